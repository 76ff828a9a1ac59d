"""GPU parity of wkv_forward_host (host-resident k, v and out streamed through
the device in segments) against the float64 oracle, element by element, at
the bars of parity_util: several segments and a ragged last one, batch rows
copied as 2-D strided copies, bf16, the state in and out, a single segment,
and the pipeline under CUDA-graph capture.
"""
import numpy as np
import pytest
import torch

import wkv_recurrence_b200 as W
from wkv_recurrence_b200 import inputs as I
from parity_util import RTOL_BF16, RTOL_F32, assert_out, assert_state, dev_f32, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from wkv_recurrence_b200 import build
    build.build()


def _pinned(x: np.ndarray, bf16: bool = False) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x))
    if bf16:
        t = t.view(torch.int16).view(torch.bfloat16)
    return t.pin_memory()


@pytest.mark.parametrize("shape,seg", [((1, 5000, 64), 1000), ((3, 2500, 96), 777), ((2, 4097, 128), 0),
                                       ((2, 300, 64), 300), ((1, 65, 32), 64)],
                         ids=["5seg", "ragged_batched", "auto", "one_seg", "two_seg"])
@pytest.mark.parametrize("with_state", [False, True], ids=["nostate", "state"])
def test_forward_host_matches_oracle(oracle, shape, seg, with_state):
    B, T, C = shape
    k, v, w, u, st = I.random_case(B, T, C, seed=B * 13 + T + C, k_spike=30.0, w_range=(1e-4, 8.0),
                                   state=with_state)
    S = None if st is None else tuple(dev_f32(x) for x in st)
    out, so = W.forward_host(_pinned(k), _pinned(v), dev_f32(w), dev_f32(u), S, seg_tokens=seg)
    torch.cuda.synchronize()
    ref, rst = oracle.recurrence_forward(k, v, w, u, st)
    sc, sst = oracle.abs_scale_forward(k, v, w, u, st)
    assert_out(out.numpy(), ref, sc, RTOL_F32)
    assert_state(tuple(host(x) for x in so), rst, sst[0], RTOL_F32)


@pytest.mark.parametrize("out_dtype", ["bf16", "f32"])
def test_forward_host_bf16(oracle, out_dtype):
    B, T, C = 2, 3000, 128
    k, v, w, u, st = I.random_case(B, T, C, seed=71, k_scale=3.0, state=True)
    kb, vb = I.f32_to_bf16_bits(k), I.f32_to_bf16_bits(v)
    od = torch.bfloat16 if out_dtype == "bf16" else torch.float32
    S = tuple(dev_f32(x) for x in st)
    out, so = W.forward_host(_pinned(kb, True), _pinned(vb, True), dev_f32(w), dev_f32(u), S, out_dtype=od,
                             seg_tokens=700)
    torch.cuda.synchronize()
    ref, rst = oracle.recurrence_forward(kb, vb, w, u, st, kv_dtype="bf16")
    sc, sst = oracle.abs_scale_forward(kb, vb, w, u, st, kv_dtype="bf16")
    assert_out(out.float().numpy(), ref, sc, RTOL_BF16, out_dtype == "bf16")
    assert_state(tuple(host(x) for x in so), rst, sst[0], RTOL_BF16)


def test_forward_host_calls_in_a_row_and_in_a_graph(oracle):
    """The library's copy streams fork from the current stream and join it:
    calls in a row reuse the buffer, and a captured call replays correctly."""
    B, T, C = 2, 3000, 64
    k, v, w, u, st = I.random_case(B, T, C, seed=83, k_spike=30.0, state=True)
    K, V = _pinned(k), _pinned(v)
    Wt, U = dev_f32(w), dev_f32(u)
    S = tuple(dev_f32(x) for x in st)
    ref, rst = oracle.recurrence_forward(k, v, w, u, st)
    sc, sst = oracle.abs_scale_forward(k, v, w, u, st)
    out = torch.empty(B, T, C).pin_memory()
    so = tuple(torch.empty(B, C, device="cuda") for _ in range(3))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for _ in range(3):
            W.forward_host(K, V, Wt, U, S, out=out, state_out=so, seg_tokens=512)
    torch.cuda.synchronize()
    assert_out(out.numpy(), ref, sc, RTOL_F32)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        W.forward_host(K, V, Wt, U, S, out=out, state_out=so, seg_tokens=512)
    out.fill_(float("nan"))
    for x in so:
        x.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    assert_out(out.numpy(), ref, sc, RTOL_F32)
    assert_state(tuple(host(x) for x in so), rst, sst[0], RTOL_F32)


def test_forward_host_rejects_bad_arguments():
    k = torch.zeros(1, 10, 64)
    w = torch.zeros(64, device="cuda")
    with pytest.raises(ValueError):
        W.forward_host(k.cuda(), k.cuda(), w, w)  # device tensors: not the host entry point's
    with pytest.raises(ValueError):
        W.forward_host(k, k, w, torch.zeros(32, device="cuda"))
    small = torch.zeros(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(W.WkvError) as e:
        W.forward_host(k, k, w, w, buffer=small)
    assert e.value.code == 4  # WKV_ERR_WORKSPACE_TOO_SMALL
