"""wkv_forward_noalloc: the forward entry point that allocates nothing.

Some callers cannot allocate device memory: a host application whose own pool
owns the whole GPU and hands a plug-in only its inputs and outputs, or code
with hard latency limits that cannot take the device-wide synchronisation of
cudaMalloc. For them the library keeps its scratch in a fixed device array.
This test calls that entry point through the C ABI, twice in a row on
different inputs, and checks each result against the ordinary wkv_forward
(which takes a caller-allocated workspace). Collected last on purpose: if it
fails, every other test has already run.
"""
import ctypes

import numpy as np
import pytest
import torch

import wkv_recurrence_b200 as W
from wkv_recurrence_b200 import _abi
from wkv_recurrence_b200 import inputs as I
from parity_util import RTOL_F32, assert_out, dev_f32, host

pytestmark = pytest.mark.gpu


def _noalloc(L, K, V, Wt, U, out, state_in=None, state_out=None):
    B, T, C = K.shape
    sin = _abi.wkv_cstate(*(s.data_ptr() for s in state_in)) if state_in is not None else None
    sout = _abi.wkv_state(*(s.data_ptr() for s in state_out)) if state_out is not None else None
    return L.wkv_forward_noalloc(B, T, C, ctypes.c_void_p(K.data_ptr()), ctypes.c_void_p(V.data_ptr()),
                                 _abi.WKV_F32, ctypes.c_void_p(Wt.data_ptr()), ctypes.c_void_p(U.data_ptr()),
                                 ctypes.c_void_p(out.data_ptr()), _abi.WKV_F32,
                                 ctypes.byref(sin) if sin is not None else None,
                                 ctypes.byref(sout) if sout is not None else None,
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_forward_on_two_calls(oracle):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from wkv_recurrence_b200 import build
    build.build()
    L = _abi.lib()
    cases = [(4, 1000, 256, True), (3, 2049, 192, False)]  # both take the chunked-scan kernel
    for call, (B, T, C, with_state) in enumerate(cases):
        k, v, w, u, st = I.random_case(B, T, C, seed=500 + call, k_spike=30.0, w_range=(1e-4, 8.0),
                                       state=with_state)
        assert W.workspace_size(B, T, C) > 256  # scratch beyond the header is in use
        K, V, Wt, U = dev_f32(k), dev_f32(v), dev_f32(w), dev_f32(u)
        S = None if st is None else tuple(dev_f32(s) for s in st)
        out = torch.full((B, T, C), float("nan"), device="cuda")
        so = tuple(torch.full((B, C), float("nan"), device="cuda") for _ in range(3))
        assert _noalloc(L, K, V, Wt, U, out, S, so) == _abi.WKV_OK
        ref_out, ref_state = W.forward(K, V, Wt, U, S)
        torch.cuda.synchronize()
        sc, sst = oracle.abs_scale_forward(k, v, w, u, st)
        assert_out(host(out), host(ref_out), sc, RTOL_F32, what=f"noalloc call {call + 1}")
        for a, b in zip(so, ref_state):
            assert np.allclose(host(a), host(b), rtol=RTOL_F32, atol=0)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = _abi.lib()
    B, T, C = 1, 1 << 20, 2048  # needs far more than the fixed array holds
    assert W.workspace_size(B, T, C) > _abi.NOALLOC_SCRATCH_BYTES
    x = ctypes.c_void_p(0x1000)  # never dereferenced: rejected before any launch
    code = L.wkv_forward_noalloc(B, T, C, x, x, _abi.WKV_F32, x, x, x, _abi.WKV_F32, None, None, None)
    assert code == _abi.WKV_ERR_WORKSPACE_TOO_SMALL
