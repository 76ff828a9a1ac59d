"""GPU parity of the cluster scan (kernel 5) and of the two optional inputs of
the RWKV-v6 time-mixing block ("RWKV-v6 Architecture: Attention-Free Linear
Transformers"): per-token decays w_t (section "2. Dynamic Data-Dependent
Decay") and the receptance gate out = sigmoid(r) * wkv. Everything through
the C ABI's wkv_forward_ext / wkv_step_ext, against the float64 oracle,
element by element, at the bars of parity_util.
"""
import numpy as np
import pytest
import torch

import wkv_recurrence_b200 as W
from wkv_recurrence_b200 import inputs as I
from parity_util import (RTOL_BF16, RTOL_F32, assert_out, assert_state, dev_bf16, dev_f32, host)

pytestmark = pytest.mark.gpu

SEQ, CHUNK, TWO, PIPE, CLUSTER = ({"kernel": k} for k in (1, 2, 3, 4, 5))


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from wkv_recurrence_b200 import build
    build.build()


def _wt(shape, seed, lo=-1.0, sigma=1.0):
    g = np.random.default_rng(seed)
    return np.clip(np.exp(g.normal(lo, sigma, shape)), 1e-4, 8.0).astype(np.float32)


def _r(shape, seed):
    return np.random.default_rng(seed + 1).normal(0.0, 2.0, shape).astype(np.float32)


def run_ext(k, v, w, u, state=None, kv="f32", out_dtype=None, options=None, w_t=None, r=None, aligned=True):
    K = dev_bf16(k) if kv == "bf16" else dev_f32(k)
    V = dev_bf16(v) if kv == "bf16" else dev_f32(v)
    if not aligned:  # base addresses 4 bytes past a 16-byte boundary: no TMA
        K = dev_f32(np.concatenate([[0.0], k.ravel()]).astype(np.float32))[1:].view(*k.shape)
        V = dev_f32(np.concatenate([[0.0], v.ravel()]).astype(np.float32))[1:].view(*v.shape)
    st = None if state is None else tuple(dev_f32(s) for s in state)
    od = {"f32": torch.float32, "bf16": torch.bfloat16, None: None}[out_dtype]
    R = None
    if r is not None:
        R = dev_bf16(r) if kv == "bf16" else dev_f32(r)
    ws = W.make_workspace(*k.shape, options=options)
    out, so = W.forward(K, V, None if w_t is not None else dev_f32(w), dev_f32(u), st, out_dtype=od,
                        workspace=ws, options=options, w_t=None if w_t is None else dev_f32(w_t), r=R)
    assert W.query_status(ws) == 0
    return host(out), tuple(host(s) for s in so)


def compare_ext(oracle, k, v, w, u, state=None, kv="f32", out_dtype=None, options=None, w_t=None, r=None,
                rtol=None, aligned=True):
    out, st = run_ext(k, v, w, u, state, kv, out_dtype, options, w_t, r, aligned)
    ref, rst = oracle.recurrence_forward(k, v, w, u, state, kv_dtype=kv, w_t=w_t, r=r)
    sc, sst = oracle.abs_scale_forward(k, v, w, u, state, kv_dtype=kv, w_t=w_t, r=r)
    rtol = rtol or (RTOL_BF16 if kv == "bf16" else RTOL_F32)
    eo = assert_out(out, ref, sc, rtol, (out_dtype or kv) == "bf16")
    es = assert_state(st, rst, sst[0], rtol)
    return eo, es


# ---------------------------------------------------------------------------
# the cluster scan
# ---------------------------------------------------------------------------

CLUSTER_OPTS = [CLUSTER, {"kernel": 5, "cta_warps": 4}, {"kernel": 5, "span": 32},
                {"kernel": 5, "span": 32, "cta_warps": 4}]
CLUSTER_IDS = ["w8j64", "w4j64", "w8j32", "w4j32"]


@pytest.mark.parametrize("opts", CLUSTER_OPTS, ids=CLUSTER_IDS)
@pytest.mark.parametrize("shape", [(1, 1, 64), (2, 65, 64), (3, 1000, 96), (2, 517, 200), (1, 1024, 36),
                                   (2, 2100, 64), (1, 9000, 40), (3, 4500, 200)],
                         ids=lambda s: "x".join(map(str, s)))
def test_cluster_random_f32(oracle, opts, shape):
    """One segment (T up to 2 CTAs' worth) and several (the look-back between
    segments), ragged spans, ragged channel groups."""
    B, T, C = shape
    k, v, w, u, st = I.random_case(B, T, C, seed=B * 7 + T + C, k_scale=2.0, k_spike=30.0,
                                   w_range=(1e-4, 8.0), state=(T % 2 == 1))
    compare_ext(oracle, k, v, w, u, st, options=opts)


def test_cluster_segment_boundaries(oracle):
    """T at, just below and just above multiples of a segment (2 CTAs x 8
    spans x 64 tokens = 1024 tokens for the default shape) and of a ring
    stage (16 tokens)."""
    for T in (1023, 1024, 1025, 2047, 2048, 2049, 4095, 4096, 4097, 8192, 8193, 12287, 1040, 1041, 1055):
        k, v, w, u, st = I.random_case(2, T, 64, seed=T, k_spike=40.0, w_range=(1e-4, 4.0), state=True)
        compare_ext(oracle, k, v, w, u, st, options=CLUSTER)


def test_cluster_misaligned_inputs(oracle):
    """Inputs that TMA cannot address: the call takes the single-launch scan."""
    k, v, w, u, st = I.random_case(2, 2500, 64, seed=91, k_spike=30.0, state=True)
    compare_ext(oracle, k, v, w, u, st, options=CLUSTER, aligned=False)


@pytest.mark.parametrize("out_dtype", ["bf16", "f32"])
def test_cluster_bf16(oracle, out_dtype):
    k, v, w, u, st = I.random_case(3, 1500, 128, seed=5, k_scale=4.0, state=True)
    kb, vb = I.f32_to_bf16_bits(2.0 * k), I.f32_to_bf16_bits(v)
    compare_ext(oracle, kb, vb, w, u, st, kv="bf16", out_dtype=out_dtype, options=CLUSTER,
                rtol=RTOL_BF16 if out_dtype == "bf16" else 1e-4)


def test_cluster_in_place_state_and_determinism(oracle):
    k, v, w, u, st = I.random_case(4, 1800, 96, seed=19, k_spike=50.0, state=True)
    S = tuple(dev_f32(s) for s in st)
    K, V, Wt, U = dev_f32(k), dev_f32(v), dev_f32(w), dev_f32(u)
    out, so = W.forward(K, V, Wt, U, S, state_out=S, options=CLUSTER)
    ref, rst = oracle.recurrence_forward(k, v, w, u, st)
    sc, sst = oracle.abs_scale_forward(k, v, w, u, st)
    assert_out(host(out), ref, sc, RTOL_F32)
    assert_state(tuple(host(s) for s in S), rst, sst[0], RTOL_F32)
    a, sa = W.forward(K, V, Wt, U, tuple(dev_f32(s) for s in st), options=CLUSTER)
    b, sb = W.forward(K, V, Wt, U, tuple(dev_f32(s) for s in st), options=CLUSTER)
    assert torch.equal(a, b) and all(torch.equal(x, y) for x, y in zip(sa, sb))


@pytest.mark.parametrize("name", ["layer", "long"])
def test_cluster_workload_full_size(oracle, name):
    """The cluster scan on the layer (one segment per channel group) and long
    (64 chained segments, 1% key spikes of +-U(20, 60)) workloads: every output
    and the final state against the float64 oracle."""
    wl = I.WORKLOADS[name]
    k, v = I.draw_kv(wl)
    w, u = I.draw_w(wl), I.draw_u(wl)
    st = I.draw_state(wl)
    eo, es = compare_ext(oracle, k, v, w, u, st, kv=wl.kv_dtype, out_dtype=wl.out_dtype, options=CLUSTER)
    print(f"{name} on the cluster scan: max normalised out error {eo:.2e}, state errors {es}")


def test_cluster_mixed_full_size(oracle):
    """The cluster scan on the mixed workload (16 x 4096 x 4096, bf16 k, v and
    out, a state in): every output and the final state against the oracle."""
    wl = I.WORKLOADS["mixed"]
    k, v = I.draw_kv(wl)
    w, u = I.draw_w(wl), I.draw_u(wl)
    st = I.draw_state(wl)
    eo, es = compare_ext(oracle, k, v, w, u, st, kv=wl.kv_dtype, out_dtype=wl.out_dtype, options=CLUSTER)
    print(f"mixed on the cluster scan: max normalised out error {eo:.2e}, state errors {es}")


def test_concurrent_calls_on_two_streams(oracle):
    """Calls with their own workspaces on two streams at once (the three-launch
    and the cluster scans, whose workspaces carry counters and flags): each
    result equals the oracle's."""
    cases = []
    for i, opts in enumerate((TWO, CLUSTER)):
        k, v, w, u, st = I.random_case(2, 3000 + 500 * i, 128, seed=90 + i, k_spike=30.0, state=True)
        cases.append((k, v, w, u, st, opts))
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = []
    dev_in = [(dev_f32(k), dev_f32(v), dev_f32(w), dev_f32(u), tuple(dev_f32(x) for x in st), o)
              for k, v, w, u, st, o in cases]
    torch.cuda.synchronize()
    for _ in range(3):
        outs = []
        for s, (K, V, Wt, U, S, o) in zip(streams, dev_in):
            with torch.cuda.stream(s):
                ws = W.make_workspace(*K.shape, options=o)
                outs.append(W.forward(K, V, Wt, U, S, workspace=ws, options=o))
        torch.cuda.synchronize()
    for (k, v, w, u, st, _), (out, so) in zip(cases, outs):
        ref, rst = oracle.recurrence_forward(k, v, w, u, st)
        sc, sst = oracle.abs_scale_forward(k, v, w, u, st)
        assert_out(host(out), ref, sc, RTOL_F32)
        assert_state(tuple(host(x) for x in so), rst, sst[0], RTOL_F32)


def test_automatic_choice_for_few_channels():
    """Few channels: the three-launch scan while k and v fit in L2, the
    cluster scan beyond (more than 2^24 elements of k)."""
    assert W.forward_kernel(8, 1024, 768) == 3
    assert W.forward_kernel(1, 8192, 2048) == 3
    assert W.forward_kernel(1, 8193, 2048) == 5
    assert W.forward_kernel(1, 65536, 2048) == 5
    assert W.forward_kernel(1, 65536, 2048, torch.bfloat16) == 5
    assert W.forward_kernel(16, 4096, 4096, torch.bfloat16) == 1


# ---------------------------------------------------------------------------
# per-token decay w_t
# ---------------------------------------------------------------------------

WT_KERNELS = [SEQ, CLUSTER, TWO, None, {"kernel": 5, "cta_warps": 4, "span": 32},
              {"kernel": 3, "chunk_len": 64, "scan_segments": 4}, {"kernel": 3, "chunk_len": 128, "replay_chunks": 2},
              {"kernel": 3, "chunk_len": 32, "scan_segments": 16}]
WT_IDS = ["seq", "cluster", "two", "auto", "cluster_w4j32", "two64seg4", "two128r2", "two32seg16"]


@pytest.mark.parametrize("opts", WT_KERNELS, ids=WT_IDS)
@pytest.mark.parametrize("shape", [(2, 33, 64), (3, 1000, 96), (2, 517, 200), (1, 2048, 64), (1, 4500, 64)],
                         ids=lambda s: "x".join(map(str, s)))
def test_per_token_decay(oracle, opts, shape):
    B, T, C = shape
    k, v, w, u, st = I.random_case(B, T, C, seed=T + C, k_scale=2.0, k_spike=30.0, state=(T % 2 == 1))
    compare_ext(oracle, k, v, w, u, st, options=opts, w_t=_wt(k.shape, T + C))


@pytest.mark.parametrize("opts", [SEQ, CLUSTER, TWO], ids=["seq", "cluster", "two"])
def test_per_token_decay_long_memory_and_spikes(oracle, opts):
    """Small decays (long memory, the compensated decay sums matter) and keys
    of +-60, with a state in."""
    k, v, w, u, st = I.random_case(2, 2000, 64, seed=61, k_spike=60.0, state=True)
    wt = np.exp(np.random.default_rng(61).uniform(np.log(1e-4), np.log(0.05), k.shape)).astype(np.float32)
    compare_ext(oracle, k, v, w, u, st, options=opts, w_t=wt)


@pytest.mark.parametrize("opts", [SEQ, CLUSTER, TWO], ids=["seq", "cluster", "two"])
def test_per_token_decay_bf16(oracle, opts):
    k, v, w, u, st = I.random_case(2, 900, 128, seed=7, k_scale=3.0, state=True)
    kb, vb = I.f32_to_bf16_bits(k), I.f32_to_bf16_bits(v)
    compare_ext(oracle, kb, vb, w, u, st, kv="bf16", out_dtype="bf16", options=opts, w_t=_wt(k.shape, 7))


def test_per_token_decay_plain_loads(oracle):
    """Misaligned k and v (no TMA): the sequential kernel's plain-load path."""
    k, v, w, u, st = I.random_case(2, 300, 64, seed=71, state=True)
    compare_ext(oracle, k, v, w, u, st, w_t=_wt(k.shape, 71), aligned=False)


def test_per_token_decay_constant_equals_per_channel(oracle):
    """w_t = w at every token gives the per-channel results (to rounding)."""
    k, v, w, u, st = I.random_case(2, 700, 64, seed=73, state=True)
    a, sa = run_ext(k, v, w, u, st, options=CLUSTER)
    b, sb = run_ext(k, v, w, u, st, options=CLUSTER, w_t=np.broadcast_to(w, k.shape).copy())
    sc, _ = oracle.abs_scale_forward(k, v, w, u, st)
    assert np.all(np.abs(a - b) <= 2 * RTOL_F32 * sc)


def test_per_token_decay_split_and_resume(oracle):
    k, v, w, u, st = I.random_case(2, 1500, 96, seed=75, k_spike=40.0, state=True)
    wt = _wt(k.shape, 75)
    o1, s1 = run_ext(k[:, :611], v[:, :611], w, u, st, options=CLUSTER, w_t=wt[:, :611])
    o2, s2 = run_ext(k[:, 611:], v[:, 611:], w, u, tuple(np.asarray(x, np.float32) for x in s1), options=SEQ,
                     w_t=wt[:, 611:])
    ref, rst = oracle.recurrence_forward(k, v, w, u, st, w_t=wt)
    sc, sst = oracle.abs_scale_forward(k, v, w, u, st, w_t=wt)
    assert_out(np.concatenate([o1, o2], 1), ref, sc, RTOL_F32)
    assert_state(s2, rst, sst[0], RTOL_F32)


def test_per_token_decay_refused_by_look_back_kernels():
    k, v, w, u, _ = I.random_case(1, 300, 64, seed=1)
    for opts in (CHUNK, PIPE):
        with pytest.raises(W.WkvError) as e:
            run_ext(k, v, w, u, options=opts, w_t=_wt(k.shape, 1))
        assert e.value.code == 1


# ---------------------------------------------------------------------------
# the receptance gate
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("opts", [SEQ, CHUNK, TWO, PIPE, CLUSTER, {"kernel": 1, "seq_vec": 2}],
                         ids=["seq", "chunk", "two", "pipe", "cluster", "seq_vec2"])
def test_gate(oracle, opts):
    k, v, w, u, st = I.random_case(2, 1000, 128, seed=81, k_spike=30.0, state=True)
    compare_ext(oracle, k, v, w, u, st, options=opts, r=_r(k.shape, 81))


@pytest.mark.parametrize("opts", [SEQ, CLUSTER, TWO], ids=["seq", "cluster", "two"])
def test_gate_bf16_and_ragged(oracle, opts):
    k, v, w, u, st = I.random_case(2, 777, 200, seed=83, k_scale=3.0, state=True)
    kb, vb = I.f32_to_bf16_bits(k), I.f32_to_bf16_bits(v)
    rb = I.f32_to_bf16_bits(_r(k.shape, 83))
    compare_ext(oracle, kb, vb, w, u, st, kv="bf16", out_dtype="bf16", options=opts, r=rb)


@pytest.mark.parametrize("opts", [SEQ, CLUSTER, TWO], ids=["seq", "cluster", "two"])
def test_gate_with_per_token_decay(oracle, opts):
    k, v, w, u, st = I.random_case(3, 1100, 64, seed=85, k_spike=30.0, state=True)
    compare_ext(oracle, k, v, w, u, st, options=opts, w_t=_wt(k.shape, 85), r=_r(k.shape, 85))


# ---------------------------------------------------------------------------
# decode with w_t and r
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("vec", [True, False], ids=["vector", "scalar"])
def test_step_ext_matches_oracle_and_forward(oracle, vec):
    S, C, T = 40, 64 if vec else 63, 30
    k, v, w, u, st = I.random_case(S, T, C, seed=87, state=True)
    wt, r = _wt(k.shape, 87), _r(k.shape, 87)
    state = tuple(dev_f32(s) for s in st)
    ref_state = tuple(s.astype(np.float64) for s in st)
    abs_state = (np.abs(st[0]).astype(np.float64), st[1].astype(np.float64), st[2].astype(np.float64))
    outs = []
    for t in range(T):
        o, state = W.step(state, dev_f32(k[:, t]), dev_f32(v[:, t]), None, dev_f32(u),
                          w_t=dev_f32(wt[:, t]), r=dev_f32(r[:, t]))
        ro, ref_state = oracle.recurrence_step(ref_state, k[:, t], v[:, t], wt[:, t], u, r=r[:, t])
        so, abs_state = oracle.abs_scale_step(abs_state, k[:, t], v[:, t], wt[:, t], u, r=r[:, t])
        assert_out(host(o), ro, so, RTOL_F32, what=f"step {t}")
        outs.append(host(o))
    assert_state(tuple(host(s) for s in state), ref_state, abs_state[0], RTOL_F32)
    fo, _ = run_ext(k, v, w, u, st, options=SEQ, w_t=wt, r=r)
    sc, _ = oracle.abs_scale_forward(k, v, w, u, st, w_t=wt, r=r)
    assert np.all(np.abs(np.stack(outs, 1) - fo) <= 4 * RTOL_F32 * sc)


# ---------------------------------------------------------------------------
# full-size workloads with the v6 inputs
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["layer", "long", "mixed"])
def test_workload_full_size_with_decay_and_gate(oracle, name):
    """The layer, long and mixed workloads with per-token decays drawn from the
    workload's w distribution (log-uniform [1e-4, 4] for long) and
    r ~ N(0, 1): every output and state against the float64 oracle."""
    wl = I.WORKLOADS[name]
    k, v = I.draw_kv(wl)
    u = I.draw_u(wl)
    w = I.draw_w(wl)
    st = I.draw_state(wl)
    wt = I.draw_wt_rows(wl, range(wl.B))
    r = I.draw_r_rows(wl, range(wl.B))
    eo, es = compare_ext(oracle, k, v, w, u, st, kv=wl.kv_dtype, out_dtype=wl.out_dtype, w_t=wt, r=r)
    print(f"{name} with w_t and r: max normalised out error {eo:.2e}, state errors {es}")
