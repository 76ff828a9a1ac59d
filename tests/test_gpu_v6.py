"""GPU parity of wkv_v6_forward (the RWKV-v6 matrix-valued state, "RWKV-v6
Architecture", section "3. Matrix-Valued Hidden State") against the float64
oracle, element by element.

Metric: |y - ref| <= rtol * scale with scale = sigmoid(r_t) (S^abs_t |k_t|),
the readout of the recurrence run on magnitudes (the sum of |terms|); the
state likewise against S^abs. rtol = 1e-5 for fp32 inputs; bf16 inputs with
bf16 outputs: half a bf16 ulp of the exact result plus 2e-3.
"""
import numpy as np
import pytest
import torch

import wkv_recurrence_b200 as W
from oracle import v6_oracle as V
from wkv_recurrence_b200 import inputs as I
from parity_util import RTOL_BF16, RTOL_F32, assert_out, dev_bf16, dev_f32, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from wkv_recurrence_b200 import build
    build.build()


def _case(B, T, H, D, seed, state=False):
    g = np.random.default_rng(seed)
    r = g.normal(0, 1.5, (B, T, H, D)).astype(np.float32)
    w = np.exp(-np.exp(g.normal(-1, 1.5, (B, T, H, D)))).astype(np.float32)
    k = g.normal(0, 1, (B, T, H, D)).astype(np.float32)
    v = g.normal(0, 1, (B, T, H, D)).astype(np.float32)
    s = g.normal(0, 1, (B, H, D, D)).astype(np.float32) if state else None
    return r, w, k, v, s


def run_v6(r, w, k, v, s=None, kv="f32", out_dtype=None):
    dev = dev_bf16 if kv == "bf16" else dev_f32
    od = {"f32": torch.float32, "bf16": torch.bfloat16, None: None}[out_dtype]
    y, so = W.v6_forward(dev(r), dev_f32(w), dev(k), dev(v), None if s is None else dev_f32(s), out_dtype=od)
    torch.cuda.synchronize()
    return host(y), host(so)


def compare_v6(r, w, k, v, s=None, kv="f32", out_dtype=None, rtol=None):
    y, so = run_v6(r, w, k, v, s, kv, out_dtype)
    ref, rs = V.recurrence(r, w, k, v, s, kv_dtype=kv)
    sc, ss = V.abs_scale(r, w, k, v, s, kv_dtype=kv)
    rtol = rtol or (RTOL_BF16 if kv == "bf16" else RTOL_F32)
    e = assert_out(y, ref, sc, rtol, bf16_out=(out_dtype or kv) == "bf16", what="y")
    es = assert_out(so, rs, ss, rtol if kv == "f32" else RTOL_F32, what="state")
    return e, es


@pytest.mark.parametrize("shape", [(2, 1, 2, 64), (2, 33, 3, 64), (1, 100, 2, 32), (2, 70, 1, 128),
                                   (3, 257, 2, 64), (1, 31, 5, 64)],
                         ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("state", [False, True], ids=["zero", "state"])
def test_v6_random(shape, state):
    compare_v6(*_case(*shape, seed=sum(shape), state=state))


@pytest.mark.parametrize("out_dtype", ["bf16", "f32"])
def test_v6_bf16(out_dtype):
    r, w, k, v, s = _case(2, 300, 3, 64, seed=7, state=True)
    rb, kb, vb = (I.f32_to_bf16_bits(x) for x in (r, k, v))
    compare_v6(rb, w, kb, vb, s, kv="bf16", out_dtype=out_dtype, rtol=RTOL_BF16 if out_dtype == "bf16" else 1e-5)


def test_v6_in_place_state_split_and_determinism():
    r, w, k, v, s = _case(2, 500, 2, 64, seed=9, state=True)
    S = dev_f32(s)
    y1, _ = W.v6_forward(dev_f32(r[:, :200]), dev_f32(w[:, :200]), dev_f32(k[:, :200]), dev_f32(v[:, :200]), S,
                         state_out=S)
    y2, _ = W.v6_forward(dev_f32(r[:, 200:]), dev_f32(w[:, 200:]), dev_f32(k[:, 200:]), dev_f32(v[:, 200:]), S,
                         state_out=S)
    ref, rs = V.recurrence(r, w, k, v, s)
    sc, ss = V.abs_scale(r, w, k, v, s)
    assert_out(np.concatenate([host(y1), host(y2)], 1), ref, sc, RTOL_F32)
    assert_out(host(S), rs, ss, RTOL_F32, what="state")
    a, sa = run_v6(r, w, k, v, s)
    b, sb = run_v6(r, w, k, v, s)
    assert np.array_equal(a, b) and np.array_equal(sa, sb)


def test_v6_empty_sequence_passes_state():
    s = np.random.default_rng(1).normal(size=(2, 3, 64, 64)).astype(np.float32)
    z = torch.empty(2, 0, 3, 64, device="cuda")
    y, so = W.v6_forward(z, z, z, z, dev_f32(s))
    assert y.shape == (2, 0, 3, 64) and np.array_equal(host(so), s.astype(np.float64))


@pytest.mark.parametrize("name", ["v6", "v6_bf16"])
def test_v6_workload_full_size(name):
    wl = I.V6_WORKLOADS[name]
    r, w, k, v = I.draw_v6(wl)
    e, es = compare_v6(r, w, k, v, None, kv=wl.kv_dtype, out_dtype=wl.out_dtype)
    print(f"{name}: max normalised y error {e:.2e}, state {es:.2e}")
