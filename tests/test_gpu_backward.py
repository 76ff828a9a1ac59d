"""GPU parity of wkv_backward (through the C ABI) against the float64 oracle's
backward recurrence, element by element.

Metric: each gradient element must satisfy |gpu - ref| <= rtol * scale, where
scale is the oracle's magnitude scale of that element (the same formulas with
every signed quantity replaced by its magnitude: the sum of |terms| that make
up the gradient), the analogue of the forward's sum_i p_i |v_i|. rtol = 1e-5.
"""
import numpy as np
import pytest
import torch

import wkv_recurrence_b200 as W
from wkv_recurrence_b200 import inputs as I
from parity_util import dev_bf16, dev_f32, host

pytestmark = pytest.mark.gpu

RTOL = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from wkv_recurrence_b200 import build
    build.build()


def assert_grad(got, ref, scale, rtol, what):
    got = np.asarray(got, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    err = np.abs(got - ref) / np.maximum(scale, 1e-30)
    worst = float(err.max()) if err.size else 0.0
    if worst > rtol:
        idx = np.unravel_index(int(np.argmax(err)), err.shape)
        raise AssertionError(f"{what}: normalised error {worst:.3e} > {rtol:.0e} at {idx}: gpu {got[idx]!r} "
                             f"ref {ref[idx]!r} scale {scale[idx]!r}")
    return worst


def run_backward(k, v, w, u, g, state=None, kv="f32"):
    K = dev_bf16(k) if kv == "bf16" else dev_f32(k)
    V = dev_bf16(v) if kv == "bf16" else dev_f32(v)
    st = None if state is None else tuple(dev_f32(s) for s in state)
    dk, dv, dw, du, ds = W.backward(K, V, dev_f32(w), dev_f32(u), dev_f32(g), st)
    torch.cuda.synchronize()
    return {"dk": host(dk), "dv": host(dv), "dw": host(dw), "du": host(du),
            "dnum": host(ds[0]), "dden": host(ds[1]), "dmax": host(ds[2])}


def compare_backward(oracle, k, v, w, u, g, state=None, kv="f32", rtol=RTOL):
    got = run_backward(k, v, w, u, g, state, kv)
    ref, sc = oracle.recurrence_backward(k, v, w, u, g, state, kv_dtype=kv)
    worst = {}
    for name in ("dk", "dv", "dw", "du", "dnum", "dden", "dmax"):
        worst[name] = assert_grad(got[name], ref[name], sc[name], rtol, name)
    return worst


@pytest.mark.parametrize("shape", [(2, 1, 64), (2, 33, 64), (3, 100, 96), (2, 517, 200), (1, 2048, 64),
                                   (4, 64, 128), (1, 32, 8)],
                         ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("state", [False, True], ids=["nostate", "state"])
def test_backward_random(oracle, shape, state):
    B, T, C = shape
    k, v, w, u, st = I.random_case(B, T, C, seed=B * 3 + T + C, k_scale=2.0, k_spike=30.0, w_range=(1e-4, 8.0),
                                   state=state)
    g = np.random.default_rng(T + C).normal(size=k.shape).astype(np.float32)
    compare_backward(oracle, k, v, w, u, g, st)


def test_backward_bf16_inputs(oracle):
    k, v, w, u, st = I.random_case(2, 700, 128, seed=5, k_scale=3.0, state=True)
    kb, vb = I.f32_to_bf16_bits(k), I.f32_to_bf16_bits(v)
    g = np.random.default_rng(5).normal(size=k.shape).astype(np.float32)
    compare_backward(oracle, kb, vb, w, u, g, st, kv="bf16")


@pytest.mark.parametrize("mag", [60.0, 100.0], ids=["k60", "k100"])
def test_backward_extreme_keys(oracle, mag):
    k, v, w, u, st = I.random_case(2, 600, 64, seed=int(mag), k_spike=mag, w_range=(1e-4, 4.0), state=True)
    g = np.random.default_rng(int(mag)).normal(size=k.shape).astype(np.float32)
    compare_backward(oracle, k, v, w, u, g, st)


def test_backward_shift_invariants_on_gpu(oracle):
    """sum_t dv_t + den0 dnum0 = sum_t g_t and sum_t dk_t + dm0 = 0 (any inputs)."""
    k, v, w, u, st = I.random_case(3, 300, 64, seed=9, k_spike=20.0, state=True)
    g = np.random.default_rng(9).normal(size=k.shape).astype(np.float32)
    d = run_backward(k, v, w, u, g, st)
    _, sc = oracle.recurrence_backward(k, v, w, u, g, st)
    lhs = d["dv"].sum(axis=1) + st[1] * d["dnum"]
    tol = 4 * RTOL * (sc["dv"].sum(axis=1) + st[1] * sc["dnum"])
    assert np.all(np.abs(lhs - g.astype(np.float64).sum(axis=1)) <= tol)
    tol = 4 * RTOL * (sc["dk"].sum(axis=1) + sc["dmax"])
    assert np.all(np.abs(d["dk"].sum(axis=1) + d["dmax"]) <= tol)


def test_backward_is_deterministic():
    k, v, w, u, st = I.random_case(2, 1000, 128, seed=11, k_spike=30.0, state=True)
    g = np.random.default_rng(11).normal(size=k.shape).astype(np.float32)
    a = run_backward(k, v, w, u, g, st)
    b = run_backward(k, v, w, u, g, st)
    for name in a:
        assert np.array_equal(a[name], b[name]), name


def test_autograd_function_matches_oracle(oracle):
    """WKV.apply inside a torch graph: gradients of sum(g * wkv) reach k, v, w, u."""
    k, v, w, u, _ = I.random_case(2, 200, 64, seed=13, k_scale=2.0)
    g = np.random.default_rng(13).normal(size=k.shape).astype(np.float32)
    K, V, Wt, U = (dev_f32(x).requires_grad_() for x in (k, v, w, u))
    out = W.WKV.apply(K, V, Wt, U)
    (out * dev_f32(g)).sum().backward()
    ref, sc = oracle.recurrence_backward(k, v, w, u, g)
    for t, name in ((K, "dk"), (V, "dv"), (Wt, "dw"), (U, "du")):
        assert_grad(host(t.grad), ref[name], sc[name], RTOL, name)
    fref, _ = oracle.recurrence_forward(k, v, w, u)
    assert np.allclose(host(out.detach()), fref, rtol=1e-4, atol=1e-5)


def test_backward_rejects_bad_arguments():
    k = torch.zeros(1, 10, 64, device="cuda")
    w = torch.zeros(64, device="cuda")
    with pytest.raises(ValueError):
        W.backward(k, k, w, w, torch.zeros(1, 10, 32, device="cuda"))
    # misaligned k (no TMA for the backward's forward pass): refused
    kk = torch.zeros(10 * 64 + 1, device="cuda")[1:].view(1, 10, 64)
    with pytest.raises(W.WkvError) as e:
        W.backward(kk, kk, w, w, torch.zeros(1, 10, 64, device="cuda"))
    assert e.value.code == 3


@pytest.mark.parametrize("name", ["layer", "long"])
def test_backward_workload_full_size(oracle, name):
    """The layer (8 x 1024 x 768) and long (1 x 65536 x 2048, 1% spikes of
    +-U(20, 60), w log-uniform [1e-4, 4]) workloads with g ~ N(0, 1): every
    gradient element against the float64 oracle."""
    wl = I.WORKLOADS[name]
    k, v = I.draw_kv(wl)
    w, u = I.draw_w(wl), I.draw_u(wl)
    st = I.draw_state(wl)
    g = I.draw_r_rows(wl, range(wl.B))  # a seeded N(0, 1) stream of the workload's shape
    worst = compare_backward(oracle, k, v, w, u, g, st)
    print(f"{name} backward: max normalised errors {worst}")
