"""wkv_forward_noalloc: the forward entry point that allocates nothing.

Some callers cannot allocate device memory: a host application whose own pool
owns the whole GPU and hands a plug-in only its inputs and outputs, or code
with hard latency limits that cannot take the device-wide synchronisation of
cudaMalloc. For them the library keeps its scratch in a fixed device array.
These tests call that entry point through the C ABI several times in a row on
different inputs and check every result against the float64 oracle at the
same bar as the other parity tests, and against the ordinary wkv_forward
(which takes a caller-allocated workspace). Collected last on purpose: if one
fails, every other test has already run.
"""
import ctypes

import numpy as np
import pytest
import torch

import wkv_recurrence_b200 as W
from wkv_recurrence_b200 import _abi
from wkv_recurrence_b200 import inputs as I
from parity_util import RTOL_F32, assert_out, assert_state, dev_f32, host

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


def _offset_by_one(x: np.ndarray, shape) -> torch.Tensor:
    """A device copy of x whose base address is 4 bytes past a 16-byte boundary
    (so TMA cannot address it and the plain-load kernels run)."""
    return dev_f32(np.concatenate([[0.0], x.ravel()]).astype(np.float32))[1:].view(*shape)


def _check_call(oracle, L, B, T, C, seed, with_state, misaligned, what):
    k, v, w, u, st = I.random_case(B, T, C, seed=seed, k_spike=30.0, w_range=(1e-4, 8.0), state=with_state)
    if misaligned:
        K, V = _offset_by_one(k, (B, T, C)), _offset_by_one(v, (B, T, C))
        out = torch.full((B * T * C + 1,), float("nan"), device="cuda")[1:].view(B, T, C)
    else:
        K, V = dev_f32(k), dev_f32(v)
        out = torch.full((B, T, C), float("nan"), device="cuda")
    Wt, U = dev_f32(w), dev_f32(u)
    S = None if st is None else tuple(dev_f32(s) for s in st)
    so = tuple(torch.full((B, C), float("nan"), device="cuda") for _ in range(3))
    assert _noalloc(L, K, V, Wt, U, out, S, so) == _abi.WKV_OK
    torch.cuda.synchronize()
    # against the float64 oracle, at the same bar as every parity test
    ref, rst = oracle.recurrence_forward(k, v, w, u, st)
    sc, sst = oracle.abs_scale_forward(k, v, w, u, st)
    assert_out(host(out), ref, sc, RTOL_F32, what=what)
    assert_state(tuple(host(s) for s in so), rst, sst[0], RTOL_F32, what=what + " state")
    # and against the entry point with a caller-allocated workspace
    ref_out, ref_state = W.forward(K, V, Wt, U, S)
    torch.cuda.synchronize()
    assert_out(host(out), host(ref_out), sc, RTOL_F32, what=what + " vs wkv_forward")
    for a, b in zip(so, ref_state):
        assert np.allclose(host(a), host(b), rtol=RTOL_F32, atol=0)


def test_noalloc_matches_oracle_on_calls_in_a_row(oracle):
    """Calls in a row: the three-launch scan (chunk totals and incoming states
    in the scratch array) and misaligned inputs (the single-launch scan, whose
    flags share the array and must start from a clean epoch on every call);
    each against the oracle."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from wkv_recurrence_b200 import build
    build.build()
    L = _abi.lib()
    assert W.forward_kernel(4, 1000, 256) == 3 and W.forward_kernel(3, 9000, 192) == 3
    cases = [(4, 1000, 256, True, False), (3, 9000, 192, False, False), (2, 4097, 128, True, False),
             (2, 5000, 128, True, True), (3, 777, 64, False, True), (2, 8200, 96, False, False)]
    for call, (B, T, C, with_state, misaligned) in enumerate(cases):
        _check_call(oracle, L, B, T, C, 500 + call, with_state, misaligned,
                    f"noalloc call {call + 1} ({'misaligned' if misaligned else 'aligned'})")


def test_noalloc_runs_the_cluster_scan(oracle):
    """A shape whose k and v exceed L2 takes the cluster scan (16 chained
    segments per channel group here), whose flags live in the scratch array
    and are cleared by every call: two calls in a row, each against the
    oracle."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = _abi.lib()
    B, T, C = 1, 16384, 2048
    assert W.forward_kernel(B, T, C) == 5
    assert W.workspace_size(B, T, C) <= _abi.NOALLOC_SCRATCH_BYTES
    for call in range(2):
        _check_call(oracle, L, B, T, C, 700 + call, call == 0, False, f"noalloc cluster scan, call {call + 1}")


def test_noalloc_rejects_shapes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = _abi.lib()
    B, T, C = 1, 1 << 20, 2048  # needs far more than the fixed array holds
    assert W.workspace_size(B, T, C) > _abi.NOALLOC_SCRATCH_BYTES
    x = ctypes.c_void_p(0x1000)  # never dereferenced: rejected before any launch
    code = L.wkv_forward_noalloc(B, T, C, x, x, _abi.WKV_F32, x, x, x, _abi.WKV_F32, None, None, None)
    assert code == _abi.WKV_ERR_WORKSPACE_TOO_SMALL
