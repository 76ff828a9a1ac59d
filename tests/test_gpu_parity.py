"""GPU parity: libwkv.so (through its Python binding over the C ABI) against the
float64 CPU oracle, element by element on seeded inputs.

Sizes span several tiles and a ragged tail; every workload shape of the
benchmark suite also runs at full size (all outputs compared against the
float64 recurrence, plus sampled outputs against the direct sum of the wkv_t
equation). Metrics and tolerances: parity_util.
"""
import time

import numpy as np
import pytest
import torch

import wkv_recurrence_b200 as W
from wkv_recurrence_b200 import inputs as I
from parity_util import (RTOL_BF16, RTOL_F32, assert_out, assert_state, dev_bf16, dev_f32, host)

pytestmark = pytest.mark.gpu

SEQ = {"kernel": 1}
CHUNK = {"kernel": 2}
TWO = {"kernel": 3}
PIPE = {"kernel": 4}
KERNELS = [SEQ, CHUNK, TWO, PIPE]
KIDS = ["seq", "chunk", "two", "pipe"]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from wkv_recurrence_b200 import build
    build.build()


def run_forward(k, v, w, u, state=None, kv="f32", out_dtype=None, options=None):
    K = dev_bf16(k) if kv == "bf16" else dev_f32(k)
    V = dev_bf16(v) if kv == "bf16" else dev_f32(v)
    st = None if state is None else tuple(dev_f32(s) for s in state)
    od = {"f32": torch.float32, "bf16": torch.bfloat16, None: None}[out_dtype]
    ws = W.make_workspace(*k.shape, options=options)
    out, so = W.forward(K, V, dev_f32(w), dev_f32(u), st, out_dtype=od, workspace=ws, options=options)
    assert W.query_status(ws) == 0
    return host(out), tuple(host(s) for s in so)


def compare(oracle, k, v, w, u, state=None, kv="f32", out_dtype=None, options=None, rtol=None):
    out, st = run_forward(k, v, w, u, state, kv, out_dtype, options)
    ref, rst = oracle.recurrence_forward(k, v, w, u, state, kv_dtype=kv)
    sc, sst = oracle.abs_scale_forward(k, v, w, u, state, kv_dtype=kv)
    bf16_out = (out_dtype or kv) == "bf16"
    rtol = rtol or (RTOL_BF16 if kv == "bf16" else RTOL_F32)
    eo = assert_out(out, ref, sc, rtol, bf16_out)
    es = assert_state(st, rst, sst[0], rtol)
    return out, st, eo, es


# ---------------------------------------------------------------------------
# small cases: both kernels, ragged shapes, dtypes
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("opts", [None, SEQ, CHUNK, {"kernel": 2, "chunk_len": 32, "lookback_group": 1},
                                  {"kernel": 2, "chunk_len": 128, "lookback_group": 3},
                                  {"kernel": 2, "chunk_len": 32, "lookback_group": 5, "span": 8},
                                  {"kernel": 2, "chunk_len": 64, "span": 8},
                                  TWO, {"kernel": 3, "chunk_len": 32, "span": 8},
                                  {"kernel": 3, "chunk_len": 64},
                                  {"kernel": 3, "chunk_len": 32, "scan_segments": 4},
                                  {"kernel": 3, "chunk_len": 32, "span": 8, "scan_segments": 16},
                                  {"kernel": 3, "chunk_len": 32, "scan_segments": 64},
                                  {"kernel": 3, "chunk_len": 32, "replay_chunks": 2},
                                  {"kernel": 3, "chunk_len": 64, "scan_segments": 4, "replay_chunks": 4},
                                  {"kernel": 3, "chunk_len": 32, "seq_threads": 64},
                                  {"kernel": 3, "chunk_len": 64, "seq_threads": 128, "replay_chunks": 2},
                                  PIPE, {"kernel": 4, "chunk_len": 32, "lookback_group": 1},
                                  {"kernel": 4, "chunk_len": 64, "span": 8, "stages": 2},
                                  {"kernel": 4, "chunk_len": 64, "span": 8, "lookback_group": 3, "stages": 5},
                                  {"kernel": 4, "chunk_len": 32, "span": 8, "lookback_group": 5, "stages": 8}],
                         ids=["auto", "seq", "chunk128", "chunk32g1", "chunk128g3", "chunk32g5s8", "chunk64s8",
                              "two128", "two32s8", "two64", "two32seg4", "two32s8seg16", "two32seg64", "two32r2", "two64seg4r4", "two32t64", "two64t128r2", "pipe128", "pipe32g1", "pipe64s8st2",
                              "pipe64s8g3st5", "pipe32s8g5st8"])
@pytest.mark.parametrize("shape", [(1, 1, 64), (2, 33, 64), (3, 1000, 128), (2, 517, 200), (1, 2048, 64)],
                         ids=lambda s: "x".join(map(str, s)))
def test_random_f32(oracle, opts, shape):
    B, T, C = shape
    k, v, w, u, st = I.random_case(B, T, C, seed=B * 1000 + T + C, k_scale=2.0, k_spike=30.0,
                                   w_range=(1e-4, 8.0), state=(T % 2 == 1))
    compare(oracle, k, v, w, u, st, options=opts)


@pytest.mark.parametrize("opts", KERNELS, ids=KIDS)
@pytest.mark.parametrize("C", [1, 5, 127, 130])
def test_ragged_channels_plain_load_path(oracle, opts, C):
    """C * 4 bytes not a multiple of 16: the kernels fill tiles with plain loads."""
    k, v, w, u, st = I.random_case(2, 300, C, seed=C, state=True)
    compare(oracle, k, v, w, u, st, options=opts)


@pytest.mark.parametrize("opts", KERNELS, ids=KIDS)
def test_misaligned_pointers(oracle, opts):
    B, T, C = 2, 257, 64
    k, v, w, u, _ = I.random_case(B, T, C, seed=77)
    K = dev_f32(np.concatenate([[0.0], k.ravel()]))[1:].view(B, T, C)
    V = dev_f32(np.concatenate([[0.0], v.ravel()]))[1:].view(B, T, C)
    out = torch.empty(B * T * C + 1, device="cuda")[1:].view(B, T, C)
    ws = W.make_workspace(B, T, C, options=opts)
    W.forward(K, V, dev_f32(w), dev_f32(u), out=out, workspace=ws, options=opts)
    ref, _ = oracle.recurrence_forward(k, v, w, u)
    sc, _ = oracle.abs_scale_forward(k, v, w, u)
    assert_out(host(out), ref, sc, RTOL_F32)


@pytest.mark.parametrize("out_dtype", ["bf16", "f32"])
@pytest.mark.parametrize("opts", KERNELS, ids=KIDS)
def test_bf16_inputs(oracle, out_dtype, opts):
    k, v, w, u, st = I.random_case(2, 700, 128, seed=5, k_scale=4.0, state=True)
    kb, vb = I.f32_to_bf16_bits(2.0 * k), I.f32_to_bf16_bits(v)
    rtol = RTOL_BF16 if out_dtype == "bf16" else 1e-4
    compare(oracle, kb, vb, w, u, st, kv="bf16", out_dtype=out_dtype, options=opts, rtol=rtol)


SEQ1 = [{"kernel": 1, "seq_vec": 1}, {"kernel": 1, "seq_vec": 1, "seq_threads": 64},
        {"kernel": 1, "seq_vec": 1, "seq_threads": 128}]


@pytest.mark.parametrize("opts", SEQ1, ids=["t32", "t64", "t128"])
@pytest.mark.parametrize("shape", [(2, 33, 64), (3, 1000, 128), (2, 517, 200), (1, 70, 36)],
                         ids=lambda s: "x".join(map(str, s)))
def test_sequential_one_channel_per_thread(oracle, opts, shape):
    """The sequential kernel with one channel per thread (ragged channel groups and token tails)."""
    B, T, C = shape
    k, v, w, u, st = I.random_case(B, T, C, seed=B + T + C, k_scale=2.0, k_spike=30.0, state=True)
    compare(oracle, k, v, w, u, st, options=opts)
    kb, vb = I.f32_to_bf16_bits(2.0 * k), I.f32_to_bf16_bits(v)
    compare(oracle, kb, vb, w, u, st, kv="bf16", out_dtype="bf16", options=opts)


# ---------------------------------------------------------------------------
# special cases with closed forms
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("opts", KERNELS, ids=KIDS)
def test_first_token_and_constant_v(oracle, opts):
    k, v, w, u, _ = I.random_case(1, 200, 64, seed=9, k_scale=3.0)
    v[:] = np.float32(0.625)
    out, st = run_forward(k, v, w, u, options=opts)
    assert np.allclose(out, 0.625, rtol=RTOL_F32, atol=0)
    out1, st1 = run_forward(k[:, :1], v[:, :1], w, u, options=opts)
    assert np.allclose(out1[:, 0], v[:, 0], rtol=1e-6)
    assert np.allclose(st1[0], v[:, 0], rtol=1e-6) and np.allclose(st1[1], 1.0, rtol=1e-6)
    assert np.allclose(st1[2], k[:, 0], rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("opts", KERNELS, ids=KIDS)
@pytest.mark.parametrize("mag", [60.0, 100.0, 1000.0])
def test_extreme_keys_stay_finite(oracle, opts, mag):
    k, v, w, u, st = I.random_case(2, 600, 64, seed=int(mag), k_spike=mag, w_range=(1e-4, 4.0), state=True)
    compare(oracle, k, v, w, u, st, options=opts, rtol=RTOL_F32 if mag < 200 else 1e-4)


@pytest.mark.parametrize("opts", KERNELS, ids=KIDS)
def test_large_decay_and_bonus_limits(oracle, opts):
    k, v, w, u, _ = I.random_case(1, 300, 64, seed=11, k_scale=3.0)
    w[:] = np.float32(1e4)
    compare(oracle, k, v, w, u, options=opts)
    u[:] = np.float32(1e3)
    out, _ = run_forward(k, v, w, u, options=opts)
    assert np.allclose(out, v, rtol=1e-6, atol=0)
    w[:] = 0.0
    u[:] = np.float32(-1e3)
    compare(oracle, k, v, w, u, options=opts)


@pytest.mark.parametrize("opts", KERNELS, ids=KIDS)
def test_empty_sequence(oracle, opts):
    B, C = 3, 64
    st = tuple(dev_f32(np.full((B, C), x, np.float32)) for x in (0.5, 2.0, 1.25))
    K = torch.empty(B, 0, C, device="cuda")
    out, so = W.forward(K, K, torch.ones(C, device="cuda"), torch.zeros(C, device="cuda"), st, options=opts)
    assert out.shape == (B, 0, C)
    for a, x in zip(so, (0.5, 2.0, 1.25)):
        assert torch.all(a == x)
    out, so = W.forward(K, K, torch.ones(C, device="cuda"), torch.zeros(C, device="cuda"), options=opts)
    assert torch.all(so[0] == 0) and torch.all(so[1] == 0) and torch.all(so[2] == float("-inf"))


@pytest.mark.parametrize("opts", KERNELS, ids=KIDS)
def test_empty_state_forms_are_equivalent(oracle, opts):
    """An explicit (0, 0, -inf) state behaves like no state."""
    k, v, w, u, _ = I.random_case(2, 130, 64, seed=13)
    a, sa = run_forward(k, v, w, u, None, options=opts)
    e = (np.zeros((2, 64), np.float32), np.zeros((2, 64), np.float32), np.full((2, 64), -np.inf, np.float32))
    b, sb = run_forward(k, v, w, u, e, options=opts)
    assert np.array_equal(a, b)
    for x, y in zip(sa, sb):
        assert np.array_equal(x, y)


# ---------------------------------------------------------------------------
# structure: resume from a state, step vs forward, kernels agree, determinism
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("opts", KERNELS, ids=KIDS)
def test_split_and_resume(oracle, opts):
    k, v, w, u, st = I.random_case(2, 1500, 128, seed=17, k_spike=40.0, w_range=(1e-4, 4.0), state=True)
    o1, s1 = run_forward(k[:, :611], v[:, :611], w, u, st, options=opts)
    s1f = tuple(np.asarray(x, np.float32) for x in s1)
    o2, s2 = run_forward(k[:, 611:], v[:, 611:], w, u, s1f, options=opts)
    ref, rst = oracle.recurrence_forward(k, v, w, u, st)
    sc, sst = oracle.abs_scale_forward(k, v, w, u, st)
    assert_out(np.concatenate([o1, o2], 1), ref, sc, RTOL_F32)
    assert_state(s2, rst, sst[0], RTOL_F32)


@pytest.mark.parametrize("opts", [SEQ, {"kernel": 2, "chunk_len": 32}, {"kernel": 3, "chunk_len": 32},
                                  {"kernel": 4, "chunk_len": 32}], ids=KIDS)
def test_in_place_state(oracle, opts):
    """state_out aliases state_in; the chunked kernels use many chunks here."""
    k, v, w, u, st = I.random_case(2, 1000, 128, seed=19, state=True)
    S = tuple(dev_f32(s) for s in st)
    out, so = W.forward(dev_f32(k), dev_f32(v), dev_f32(w), dev_f32(u), S, state_out=S, options=opts)
    assert all(a.data_ptr() == b.data_ptr() for a, b in zip(so, S))
    ref, rst = oracle.recurrence_forward(k, v, w, u, st)
    sc, sst = oracle.abs_scale_forward(k, v, w, u, st)
    assert_out(host(out), ref, sc, RTOL_F32)
    assert_state(tuple(host(s) for s in S), rst, sst[0], RTOL_F32)


def test_step_matches_oracle_and_forward(oracle):
    S, C, T = 37, 68, 40
    k, v, w, u, st = I.random_case(S, T, C, seed=23, state=True)
    state = tuple(dev_f32(s) for s in st)
    ref_state = tuple(s.astype(np.float64) for s in st)
    abs_state = (np.abs(st[0]).astype(np.float64), st[1].astype(np.float64), st[2].astype(np.float64))
    outs = []
    for t in range(T):
        o, state = W.step(state, dev_f32(k[:, t]), dev_f32(v[:, t]), dev_f32(w), dev_f32(u))
        ro, ref_state = oracle.recurrence_step(ref_state, k[:, t], v[:, t], w, u)
        so, abs_state = oracle.abs_scale_step(abs_state, k[:, t], v[:, t], w, u)
        assert_out(host(o), ro, so, RTOL_F32, what=f"step {t}")
        outs.append(host(o))
    assert_state(tuple(host(s) for s in state), ref_state, abs_state[0], RTOL_F32)
    fo, _ = run_forward(k, v, w, u, st)
    assert np.allclose(np.stack(outs, 1), fo, rtol=0, atol=3e-5 * np.abs(v).max())


@pytest.mark.parametrize("vec", [True, False], ids=["vector", "scalar"])
@pytest.mark.parametrize("kv", ["f32", "bf16"])
def test_step_paths_and_in_place(oracle, vec, kv):
    S, C = 50, 64 if vec else 63
    k, v, w, u, st = I.random_case(S, 3, C, seed=29, k_scale=3.0, state=True)
    if kv == "bf16":
        k, v = I.f32_to_bf16_bits(k), I.f32_to_bf16_bits(v)
        K, V = dev_bf16(k[:, 0]), dev_bf16(v[:, 0])
        kf, vf = I.bf16_bits_to_f32(k[:, 0]), I.bf16_bits_to_f32(v[:, 0])
    else:
        K, V = dev_f32(k[:, 0]), dev_f32(v[:, 0])
        kf, vf = k[:, 0], v[:, 0]
    state = tuple(dev_f32(s) for s in st)
    o, so = W.step(state, K, V, dev_f32(w), dev_f32(u), inplace=True)
    assert all(a.data_ptr() == b.data_ptr() for a, b in zip(so, state))
    ro, rst = oracle.recurrence_step(tuple(s.astype(np.float64) for s in st), kf, vf, w, u)
    sc, sst = oracle.abs_scale_step((np.abs(st[0]).astype(np.float64), st[1], st[2]), kf, vf, w, u)
    assert_out(host(o), ro, sc, RTOL_BF16 if kv == "bf16" else RTOL_F32, bf16_out=(kv == "bf16"))
    assert_state(tuple(host(s) for s in so), rst, sst[0], RTOL_F32)


def test_step_from_empty_state(oracle):
    S, C = 8, 64
    k, v, w, u, _ = I.random_case(S, 1, C, seed=31)
    e = (torch.zeros(S, C, device="cuda"), torch.zeros(S, C, device="cuda"),
         torch.full((S, C), float("-inf"), device="cuda"))
    o, st = W.step(e, dev_f32(k[:, 0]), dev_f32(v[:, 0]), dev_f32(w), dev_f32(u))
    assert np.allclose(host(o), v[:, 0], rtol=1e-6)
    assert np.allclose(host(st[0]), v[:, 0], rtol=1e-6) and np.allclose(host(st[1]), 1.0)
    assert np.array_equal(host(st[2]), k[:, 0].astype(np.float64))


def test_kernels_agree_and_are_deterministic(oracle):
    k, v, w, u, st = I.random_case(4, 3000, 192, seed=37, k_spike=50.0, w_range=(1e-4, 8.0), state=True)
    sc, _ = oracle.abs_scale_forward(k, v, w, u, st)
    a1, _ = run_forward(k, v, w, u, st, options=SEQ)
    for opts in KERNELS + [{"kernel": 2, "chunk_len": 32, "lookback_group": 3}]:
        r1, s1 = run_forward(k, v, w, u, st, options=opts)
        r2, s2 = run_forward(k, v, w, u, st, options=opts)
        assert np.array_equal(r1, r2), opts
        for x, y in zip(s1, s2):
            assert np.array_equal(x, y), opts
        assert np.all(np.abs(a1 - r1) <= 2 * RTOL_F32 * sc), opts


@pytest.mark.parametrize("T", [1000, 20], ids=["many_chunks", "one_chunk"])
def test_back_to_back_calls_see_previous_results(T):
    """Calls queued with no synchronisation, each taking the previous call's
    output as its k and its state as the state in: the launches that may
    start before the one ahead of them ends (programmatic serialization) must
    still see its results. Bitwise equal to the same calls synchronised."""
    B, C = 2, 128
    k, v, w, u, st = I.random_case(B, T, C, seed=53, state=True)
    K, V, Wt, U = dev_f32(k), dev_f32(v), dev_f32(w), dev_f32(u)
    S0 = tuple(dev_f32(s) for s in st)
    o1, s1 = W.forward(K, V, Wt, U, S0, options=TWO)
    torch.cuda.synchronize()
    o2, s2 = W.forward(o1.clone(), V, Wt, U, tuple(x.clone() for x in s1), options=TWO)
    torch.cuda.synchronize()
    for _ in range(10):
        c1, cs1 = W.forward(K, V, Wt, U, S0, options=TWO)
        c2, cs2 = W.forward(c1, V, Wt, U, cs1, options=TWO)
        c3, _ = W.forward(c2, V, Wt, U, cs2, options=TWO)
    torch.cuda.synchronize()
    assert torch.equal(c2, o2)
    for a, b in zip(cs2, s2):
        assert torch.equal(a, b)
    o3, _ = W.forward(o2, V, Wt, U, s2, options=TWO)
    torch.cuda.synchronize()
    assert torch.equal(c3, o3)


@pytest.mark.parametrize("opts", [CHUNK, TWO, PIPE], ids=["chunk", "two", "pipe"])
def test_workspace_reuse_across_shapes(oracle, opts):
    """One workspace serves successive calls of different shapes (the epoch scheme)."""
    ws = W.make_workspace(4, 4096, 256, options=opts)
    for (B, T, C) in [(4, 4096, 256), (2, 1000, 64), (4, 4096, 256), (1, 2500, 192)]:
        k, v, w, u, _ = I.random_case(B, T, C, seed=B + T + C)
        out, _ = W.forward(dev_f32(k), dev_f32(v), dev_f32(w), dev_f32(u), workspace=ws, options=opts)
        assert W.query_status(ws) == 0
        ref, _ = oracle.recurrence_forward(k, v, w, u)
        sc, _ = oracle.abs_scale_forward(k, v, w, u)
        assert_out(host(out), ref, sc, RTOL_F32)


@pytest.mark.parametrize("kernel", [2, 4, 5], ids=["chunk", "pipe", "cluster"])
def test_bounded_wait_reports_timeout_and_recovers(oracle, kernel):
    """A chunk tile (or, in the cluster scan, a segment) that never publishes:
    waiters give up after the limit, report WKV_ERR_WAIT_TIMEOUT, and the next
    call on the same workspace is correct again."""
    B, T, C = 2, 4096, 128
    k, v, w, u, _ = I.random_case(B, T, C, seed=41)
    opts = {"kernel": kernel, "chunk_len": 64, "lookback_group": 4, "wait_timeout_ns": 20_000_000,
            "inject_enable": 1, "inject_unpublished_tile": 9}
    if kernel == 5:  # segments of 2 CTAs x 4 spans x 32 tokens = 256 tokens; tickets 0-7 are segment 0
        opts = {"kernel": 5, "cta_warps": 4, "span": 32, "wait_timeout_ns": 20_000_000, "inject_enable": 1,
                "inject_unpublished_tile": 3}
    ws = W.make_workspace(B, T, C, options=opts)
    K, V, Wt, U = dev_f32(k), dev_f32(v), dev_f32(w), dev_f32(u)
    t0 = time.time()
    W.forward(K, V, Wt, U, workspace=ws, options=opts)
    assert W.query_status(ws) == 6  # WKV_ERR_WAIT_TIMEOUT
    assert time.time() - t0 < 30
    assert W.query_status(ws) == 0  # cleared by the read
    clean = dict(opts, inject_enable=0)
    out, _ = W.forward(K, V, Wt, U, workspace=ws, options=clean)
    assert W.query_status(ws) == 0
    ref, _ = oracle.recurrence_forward(k, v, w, u)
    sc, _ = oracle.abs_scale_forward(k, v, w, u)
    assert_out(host(out), ref, sc, RTOL_F32)


def test_stage_counts_in_any_order(oracle):
    """Launches of one kernel with more, fewer, then more shared-memory stages
    again (the kernel's shared-memory limit must not shrink under a later call)."""
    B, T, C = 2, 1500, 128
    k, v, w, u, _ = I.random_case(B, T, C, seed=47)
    ref, _ = oracle.recurrence_forward(k, v, w, u)
    sc, _ = oracle.abs_scale_forward(k, v, w, u)
    for stages in (5, 2, 5, 0, 2):
        out, _ = run_forward(k, v, w, u, options={"kernel": 4, "chunk_len": 64, "stages": stages})
        assert_out(out, ref, sc, RTOL_F32)
    # a ring that does not fit in one CTA's shared memory is refused, not launched
    with pytest.raises(W.WkvError) as e:
        run_forward(k, v, w, u, options={"kernel": 4, "chunk_len": 128, "span": 16, "stages": 8})
    assert e.value.code == 1  # WKV_ERR_INVALID_ARG


@pytest.mark.parametrize("opts", KERNELS, ids=KIDS)
def test_no_wait_reaches_its_limit(oracle, opts):
    """With a 0.2 s wait limit, correct calls finish far below it: no wait in
    any kernel runs to its limit on a normal run (such a wait would give
    correct results but cost the whole limit)."""
    B, T, C = 2, 3000, 128
    k, v, w, u, _ = I.random_case(B, T, C, seed=43)
    o = dict(opts, wait_timeout_ns=200_000_000)
    ws = W.make_workspace(B, T, C, options=o)
    K, V, Wt, U = dev_f32(k), dev_f32(v), dev_f32(w), dev_f32(u)
    W.forward(K, V, Wt, U, workspace=ws, options=o)
    torch.cuda.synchronize()
    for _ in range(3):
        t0 = time.perf_counter()
        W.forward(K, V, Wt, U, workspace=ws, options=o)
        torch.cuda.synchronize()
        assert time.perf_counter() - t0 < 0.1
    assert W.query_status(ws) == 0


# ---------------------------------------------------------------------------
# the benchmark workloads at full size
# ---------------------------------------------------------------------------

def _sampled_direct(oracle, k, v, w, u, out, state, kv, n, seed, scale, rtol, bf16_out=False):
    """Sampled outputs against the direct sum of the wkv_t equation."""
    B, T, C = k.shape
    g = np.random.default_rng(seed)
    for _ in range(n):
        b, t, c = int(g.integers(B)), int(g.integers(T)), int(g.integers(C))
        s = None if state is None else (state[0][b, c], state[1][b, c], state[2][b, c])
        ref = oracle.direct_output(k[b, :, c], v[b, :, c], w[c], u[c], t, s, kv_dtype=kv)
        assert_out(np.array([out[b, t, c]]), np.array([ref]), np.array([scale[b, t, c]]), rtol, bf16_out,
                   what=f"direct sum at {(b, t, c)}")


@pytest.mark.parametrize("name", ["tiny", "small", "layer", "long", "mixed"])
def test_workload_full_size(oracle, name):
    wl = I.WORKLOADS[name]
    k, v = I.draw_kv(wl)
    w, u = I.draw_w(wl), I.draw_u(wl)
    st = I.draw_state(wl)
    out, so, eo, es = compare(oracle, k, v, w, u, st, kv=wl.kv_dtype, out_dtype=wl.out_dtype)
    rtol = RTOL_BF16 if wl.kv_dtype == "bf16" else RTOL_F32
    sc, _ = oracle.abs_scale_forward(k, v, w, u, st, kv_dtype=wl.kv_dtype)
    _sampled_direct(oracle, k, v, w, u, out, st, wl.kv_dtype, 40 if wl.T > 10000 else 100, 7, sc, rtol,
                    bf16_out=wl.out_dtype == "bf16")
    print(f"{name}: max normalised out error {eo:.2e}, state errors {es}")


@pytest.mark.parametrize("name", ["layer", "long", "mixed"])
def test_workload_full_size_three_launches(oracle, name):
    """The three-launch chunked scan on the benchmark shapes."""
    wl = I.WORKLOADS[name]
    k, v = I.draw_kv(wl)
    w, u = I.draw_w(wl), I.draw_u(wl)
    st = I.draw_state(wl)
    _, _, eo, es = compare(oracle, k, v, w, u, st, kv=wl.kv_dtype, out_dtype=wl.out_dtype, options=TWO)
    print(f"{name} (three launches): max normalised out error {eo:.2e}, state errors {es}")


@pytest.mark.parametrize("name", ["layer", "long", "mixed"])
def test_workload_full_size_pipelined(oracle, name):
    """The pipelined chunked scan on the benchmark shapes, whatever the
    automatic choice of kernel is."""
    wl = I.WORKLOADS[name]
    k, v = I.draw_kv(wl)
    w, u = I.draw_w(wl), I.draw_u(wl)
    st = I.draw_state(wl)
    _, _, eo, es = compare(oracle, k, v, w, u, st, kv=wl.kv_dtype, out_dtype=wl.out_dtype, options=PIPE)
    print(f"{name} (pipelined): max normalised out error {eo:.2e}, state errors {es}")


def test_tiny_against_decimal_golden():
    from test_oracle_pins import load_golden
    k, v, w, u, ref = load_golden()
    for opts in (None, SEQ, CHUNK, TWO, PIPE):
        out, _ = run_forward(k, v, w, u, options=opts)
        assert np.allclose(out, ref, rtol=RTOL_F32, atol=RTOL_F32 * np.abs(v).max())


def test_decode_workload_full_size(oracle):
    """4096 streams x 768 channels: a 512-token prefix (wkv_forward), then 256
    one-token wkv_step calls. The float64 oracle follows every stream: the
    prefix state of all 4096 streams, every output of every one of the 256
    steps, and the final state of every stream."""
    wl = I.WORKLOADS["decode"]
    S, C = wl.B, wl.C
    w, u = I.draw_w(wl), I.draw_u(wl)
    Wt, U = dev_f32(w), dev_f32(u)
    state = tuple(torch.empty(S, C, device="cuda") for _ in range(3))
    ref_state = tuple(np.empty((S, C)) for _ in range(3))
    abs_state = tuple(np.empty((S, C)) for _ in range(3))
    # the prefix in slices of streams, to bound host memory
    slab = 256
    for s0 in range(0, S, slab):
        kp, vp = I.draw_kv_rows(wl, range(s0, s0 + slab))
        W.forward(dev_f32(kp), dev_f32(vp), Wt, U, state_out=tuple(x[s0:s0 + slab] for x in state))
        _, rst = oracle.recurrence_forward(kp, vp, w, u)
        _, ast = oracle.abs_scale_forward(kp, vp, w, u)
        for dst, a in zip(ref_state, rst):
            dst[s0:s0 + slab] = a
        for dst, a in zip(abs_state, ast):
            dst[s0:s0 + slab] = a
        del kp, vp
    torch.cuda.synchronize()
    assert_state(tuple(host(x) for x in state), ref_state, abs_state[0], RTOL_F32, "prefix state")
    out = torch.empty(S, C, device="cuda")
    worst = 0.0
    for step in range(wl.decode_steps):
        kd, vd = I.draw_decode_token(wl, step)
        W.step(state, dev_f32(kd), dev_f32(vd), Wt, U, out=out, inplace=True)
        ro, ref_state = oracle.recurrence_step(ref_state, kd, vd, w, u)
        so, abs_state = oracle.abs_scale_step(abs_state, kd, vd, w, u)
        worst = max(worst, assert_out(host(out), ro, so, RTOL_F32, what=f"decode step {step}"))
    es = assert_state(tuple(host(x) for x in state), ref_state, abs_state[0], RTOL_F32, "final state")
    print(f"decode: max normalised out error {worst:.2e} over all streams and steps, state errors {es}")
