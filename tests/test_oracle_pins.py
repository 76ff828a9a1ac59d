"""Pins for the CPU oracle (no GPU).

Each check ties the oracle to something other than itself: a hand-worked
example, values stored from 50-digit decimal arithmetic, closed forms, special
cases that reduce to a library softmax, brute force, and invariants. All of them
follow "Linear attention without writing a CUDA kernel", section "The
recurrence" (the wkv_t equation and the carried-state step).

The checks are written as functions of an implementation ``impl(k, v, w, u,
state) -> (out, (num, den, max_e))`` so that the same suite runs against the
oracle's three forms and against deliberately broken copies of the recurrence
(test_pins_catch_planted_mistakes): every planted mistake must fail a check.
"""

import math
import os

import numpy as np
import pytest
import torch

from wkv_recurrence_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "wkv_tiny_decimal.txt")


# ---------------------------------------------------------------------------
# the checks
# ---------------------------------------------------------------------------

def check_hand_worked(impl):
    """Two tokens, one channel, worked by hand.

    k = (0, ln 2), v = (1, 3), w = ln 2, u = 0. Token 1 sees only itself: 1.
    Token 2: the earlier token has weight e^{-(2-1-1)w + k_1} = 1, the current
    one e^{u + k_2} = 2, so wkv_2 = (1*1 + 2*3) / (1 + 2) = 7/3. The state after
    token 2 holds N = e^{-w} e^{k_1} v_1 + e^{k_2} v_2 = 6.5 and D = 2.5 over the
    largest exponent max(k_1 - w, k_2) = ln 2: (3.25, 1.25, ln 2).
    """
    ln2 = np.float32(math.log(2.0))
    k = np.array([0.0, ln2], np.float32).reshape(1, 2, 1)
    v = np.array([1.0, 3.0], np.float32).reshape(1, 2, 1)
    w = np.array([ln2], np.float32)
    u = np.array([0.0], np.float32)
    out, (num, den, mx) = impl(k, v, w, u, None)
    assert out[0, 0, 0] == pytest.approx(1.0, rel=1e-6)
    assert out[0, 1, 0] == pytest.approx(7.0 / 3.0, rel=1e-6)
    assert mx[0, 0] == pytest.approx(math.log(2.0), rel=1e-6)
    assert num[0, 0] == pytest.approx(3.25, rel=1e-6)
    assert den[0, 0] == pytest.approx(1.25, rel=1e-6)


def load_golden():
    rows = [ln.split() for ln in open(GOLDEN) if not ln.startswith("#")]
    B = 1 + max(int(r[0]) for r in rows)
    T = 1 + max(int(r[1]) for r in rows)
    C = 1 + max(int(r[2]) for r in rows)
    k = np.zeros((B, T, C), np.float32)
    v = np.zeros((B, T, C), np.float32)
    w = np.zeros(C, np.float32)
    u = np.zeros(C, np.float32)
    ref = np.zeros((B, T, C))
    for r in rows:
        b, t, c = int(r[0]), int(r[1]), int(r[2])
        k[b, t, c], v[b, t, c], w[c], u[c] = (np.float32(float(x)) for x in r[3:7])
        ref[b, t, c] = float(r[7])
    return k, v, w, u, ref


def check_golden_decimal(impl, tol=1e-12):
    k, v, w, u, ref = load_golden()
    out, _ = impl(k, v, w, u, None)
    assert np.abs(out - ref).max() <= tol * max(1.0, np.abs(ref).max())


def check_first_token(impl):
    """With the empty state, token 1 returns v_1 and leaves the state (v_1, 1, k_1)."""
    k, v, w, u, _ = I.random_case(2, 1, 6, 3)
    out, (num, den, mx) = impl(k, v, w, u, None)
    assert np.allclose(out[:, 0], v[:, 0], rtol=1e-14, atol=0)
    assert np.allclose(num, v[:, 0], rtol=1e-14, atol=0)
    assert np.allclose(den, 1.0, rtol=1e-14, atol=0)
    assert np.allclose(mx, k[:, 0], rtol=1e-14, atol=0)


def check_constant_v(impl):
    """A constant value stream is returned unchanged (weights sum to one)."""
    k, v, w, u, _ = I.random_case(1, 50, 5, 4, k_scale=3.0)
    v[:] = np.float32(-1.75)
    out, _ = impl(k, v, w, u, None)
    assert np.allclose(out, -1.75, rtol=1e-13, atol=0)


def check_range(impl):
    """wkv_t is a convex combination of v_1..v_t: it lies in [min, max] of them."""
    k, v, w, u, _ = I.random_case(2, 40, 7, 5, k_scale=4.0)
    out, _ = impl(k, v, w, u, None)
    lo = np.minimum.accumulate(v, axis=1)
    hi = np.maximum.accumulate(v, axis=1)
    assert np.all(out >= lo - 1e-12) and np.all(out <= hi + 1e-12)


def check_large_w(impl):
    """w = 1e4: everything but the previous and the current token vanishes."""
    k, v, w, u, _ = I.random_case(1, 30, 6, 6, k_scale=3.0)
    w[:] = np.float32(1e4)
    out, _ = impl(k, v, w, u, None)
    kd, vd, ud = k.astype(np.float64), v.astype(np.float64), u.astype(np.float64)
    a = np.exp(kd[:, :-1])                  # previous token, undecayed
    b = np.exp(ud + kd[:, 1:])              # current token with bonus
    ref = (a * vd[:, :-1] + b * vd[:, 1:]) / (a + b)
    assert np.allclose(out[:, 0], v[:, 0], rtol=1e-14)
    assert np.allclose(out[:, 1:], ref, rtol=1e-12, atol=1e-14)


def check_causal_softmax(impl):
    """w = 0, u = 0: wkv_t = softmax(k_1..k_t) . v_1..v_t (torch CPU softmax)."""
    k, v, w, u, _ = I.random_case(1, 24, 5, 7, k_scale=2.0)
    w[:] = 0.0
    u[:] = 0.0
    out, _ = impl(k, v, w, u, None)
    T = k.shape[1]
    mask = torch.ones(T, T, dtype=torch.bool).tril()
    for c in range(k.shape[2]):
        s = torch.from_numpy(k[0, :, c].astype(np.float64)).expand(T, T).clone()
        s[~mask] = -math.inf
        ref = torch.softmax(s, dim=1) @ torch.from_numpy(v[0, :, c].astype(np.float64))
        assert np.allclose(out[0, :, c], ref.numpy(), rtol=1e-12, atol=1e-14)


def check_cumulative_mean(impl):
    """k = 0, w = 0, u = 0: every token has weight one, wkv_t is the running mean."""
    _, v, w, u, _ = I.random_case(2, 33, 3, 8)
    k = np.zeros_like(v)
    w[:] = 0.0
    u[:] = 0.0
    out, _ = impl(k, v, w, u, None)
    ref = np.cumsum(v.astype(np.float64), axis=1) / np.arange(1, v.shape[1] + 1)[None, :, None]
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-14)


def check_bonus_limits(impl):
    """u = +1e3 returns v_t; u = -1e3 with w = 0 returns softmax(k_<t) . v_<t."""
    k, v, w, u, _ = I.random_case(1, 20, 4, 9)
    u[:] = np.float32(1e3)
    out, _ = impl(k, v, w, u, None)
    assert np.allclose(out, v, rtol=1e-14, atol=0)
    u[:] = np.float32(-1e3)
    w[:] = 0.0
    out, _ = impl(k, v, w, u, None)
    T = k.shape[1]
    for c in range(k.shape[2]):
        for t in range(1, T):
            p = torch.softmax(torch.from_numpy(k[0, :t, c].astype(np.float64)), 0)
            ref = float(p @ torch.from_numpy(v[0, :t, c].astype(np.float64)))
            assert out[0, t, c] == pytest.approx(ref, rel=1e-12, abs=1e-14)


def check_masked_softmax(impl):
    """Restatement as causal attention with a query-free score (torch softmax).

    score[t, i] = k_i - (t-1-i) w for i < t, u + k_t for i = t, -inf for i > t
    (1-based), and wkv = softmax(score) @ v.
    """
    k, v, w, u, _ = I.random_case(2, 48, 4, 10, k_scale=2.5)
    out, _ = impl(k, v, w, u, None)
    B, T, C = k.shape
    t = torch.arange(T, dtype=torch.float64)[:, None]
    i = torch.arange(T, dtype=torch.float64)[None, :]
    for b in range(B):
        for c in range(C):
            kc = torch.from_numpy(k[b, :, c].astype(np.float64))
            score = kc[None, :] - (t - 1 - i) * float(w[c])
            score = torch.where(i < t, score, torch.full_like(score, -math.inf))
            score[range(T), range(T)] = float(u[c]) + kc
            ref = torch.softmax(score, dim=1) @ torch.from_numpy(v[b, :, c].astype(np.float64))
            assert np.allclose(out[b, :, c], ref.numpy(), rtol=1e-12, atol=1e-14)


def check_state_closed_form(impl):
    """The state after T tokens: max_e = max_i (k_i - (T-i) w) over 1-based i,
    den = sum_i e^{k_i - (T-i) w - max_e} >= 1, num likewise with v."""
    k, v, w, u, _ = I.random_case(2, 37, 5, 11, k_scale=3.0)
    _, (num, den, mx) = impl(k, v, w, u, None)
    T = k.shape[1]
    y = k.astype(np.float64) - (T - 1 - np.arange(T))[None, :, None] * w.astype(np.float64)
    m = y.max(axis=1)
    e = np.exp(y - m[:, None, :])
    assert np.allclose(mx, m, rtol=1e-13, atol=1e-13)
    assert np.allclose(den, e.sum(axis=1), rtol=1e-12)
    assert np.allclose(num, (e * v).sum(axis=1), rtol=1e-12, atol=1e-13)
    assert np.all(den >= 1.0 - 1e-15)


def check_split(impl):
    """Running T1 tokens, then the rest from the returned state, equals one pass."""
    k, v, w, u, st = I.random_case(2, 45, 6, 12, k_scale=2.0, state=True)
    out, s = impl(k, v, w, u, st)
    o1, s1 = impl(k[:, :17], v[:, :17], w, u, st)
    o2, s2 = impl(k[:, 17:], v[:, 17:], w, u, s1)
    assert np.allclose(np.concatenate([o1, o2], 1), out, rtol=1e-12, atol=1e-13)
    # compare states through representation-free quantities
    assert np.allclose(s2[2] + np.log(s2[1]), s[2] + np.log(s[1]), rtol=0, atol=1e-12)
    assert np.allclose(s2[0] / s2[1], s[0] / s[1], rtol=1e-12, atol=1e-13)


def check_stable_extremes(impl):
    """Keys at +-60, +-100 and +-1000 stay finite and keep the range invariant."""
    for mag in (60.0, 100.0, 1000.0):
        k, v, w, u, _ = I.random_case(1, 40, 5, 13, k_spike=mag)
        out, (num, den, mx) = impl(k, v, w, u, None)
        assert np.all(np.isfinite(out)) and np.all(np.isfinite(num)) and np.all(np.isfinite(den))
        lo = np.minimum.accumulate(v, axis=1)
        hi = np.maximum.accumulate(v, axis=1)
        assert np.all(out >= lo - 1e-12) and np.all(out <= hi + 1e-12)


ALL_CHECKS = [check_hand_worked, check_golden_decimal, check_first_token, check_constant_v,
              check_range, check_large_w, check_causal_softmax, check_cumulative_mean,
              check_bonus_limits, check_masked_softmax, check_state_closed_form, check_split,
              check_stable_extremes]


# ---------------------------------------------------------------------------
# the oracle's forms under the checks
# ---------------------------------------------------------------------------

def _recurrence(O):
    return lambda k, v, w, u, st: O.recurrence_forward(k, v, w, u, st)


def _direct(O):
    return lambda k, v, w, u, st: O.direct_forward(k, v, w, u, st)


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda f: f.__name__)
def test_recurrence_pins(oracle, check):
    check(_recurrence(oracle))


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda f: f.__name__)
def test_direct_sum_pins(oracle, check):
    check(_direct(oracle))


def test_decimal_matches_golden(oracle):
    """The 50-digit decimal sum reproduces the stored fixture (to 1e-30)."""
    k, v, w, u, ref = load_golden()
    res = oracle.decimal_forward(k, v, w, u, digits=50)
    for (b, t, c), r in np.ndenumerate(ref):
        assert abs(float(res[b][t][c]) - r) <= 1e-15 * max(1.0, abs(r))


@pytest.mark.parametrize("seed", range(6))
def test_recurrence_equals_direct_sum(oracle, seed):
    """Random cases, with and without an initial state and with large keys."""
    T = [1, 7, 33, 64, 20, 50][seed]
    k, v, w, u, st = I.random_case(2, T, 9, 100 + seed, k_scale=1.0 + seed,
                                   k_spike=[0, 0, 60, 0, 100, 30][seed],
                                   w_range=[(1e-3, 8), (1e-4, 4), (1e-4, 1e-2), (0.5, 8), (1e-3, 8), (1e-4, 4)][seed],
                                   state=bool(seed % 2))
    o1, s1 = oracle.recurrence_forward(k, v, w, u, st)
    o2, s2 = oracle.direct_forward(k, v, w, u, st)
    scale, _ = oracle.abs_scale_forward(k, v, w, u, st)
    assert np.all(np.abs(o1 - o2) <= 1e-12 * scale + 1e-300)
    assert np.allclose(s1[2] + np.log(s1[1]), s2[2] + np.log(s2[1]), rtol=0, atol=1e-12)
    assert np.allclose(s1[0] / s1[1], s2[0] / s2[1], rtol=1e-12, atol=1e-13)


def test_direct_output_matches_direct_forward(oracle):
    k, v, w, u, st = I.random_case(1, 40, 3, 21, state=True)
    out, _ = oracle.direct_forward(k, v, w, u, st)
    for t in (0, 1, 17, 39):
        for c in range(3):
            o = oracle.direct_output(k[0, :, c], v[0, :, c], w[c], u[c], t,
                                     (st[0][0, c], st[1][0, c], st[2][0, c]))
            assert o == pytest.approx(out[0, t, c], rel=1e-13, abs=1e-15)


def test_step_equals_forward(oracle):
    """T decode steps of the recurrence reproduce the sequence forward."""
    k, v, w, u, st = I.random_case(3, 25, 4, 22, state=True)
    out, s = oracle.recurrence_forward(k, v, w, u, st)
    state = tuple(x.astype(np.float64) for x in st)
    for t in range(k.shape[1]):
        o, state = oracle.recurrence_step(state, k[:, t], v[:, t], w, u)
        assert np.array_equal(o, out[:, t])
    for a, b in zip(state, s):
        assert np.array_equal(a, b)


def test_bf16_inputs_widen_exactly(oracle):
    """bf16 codes go through the oracle as the fp32 values they encode."""
    k, v, w, u, _ = I.random_case(2, 30, 5, 23, k_scale=3.0)
    kb, vb = I.f32_to_bf16_bits(k), I.f32_to_bf16_bits(v)
    o1, s1 = oracle.recurrence_forward(kb, vb, w, u, None, kv_dtype="bf16")
    o2, s2 = oracle.recurrence_forward(I.bf16_bits_to_f32(kb), I.bf16_bits_to_f32(vb), w, u, None)
    assert np.array_equal(o1, o2)
    o3, _ = oracle.direct_forward(kb, vb, w, u, None, kv_dtype="bf16")
    assert np.allclose(o1, o3, rtol=1e-12, atol=1e-13)


def test_abs_scale_bounds_output(oracle):
    k, v, w, u, st = I.random_case(2, 30, 5, 24, state=True)
    out, _ = oracle.recurrence_forward(k, v, w, u, st)
    sc, _ = oracle.abs_scale_forward(k, v, w, u, st)
    assert np.all(np.abs(out) <= sc * (1 + 1e-12))


def test_empty_sequence_passes_state(oracle):
    k = np.zeros((2, 0, 3), np.float32)
    st = tuple(np.full((2, 3), x, np.float32) for x in (0.5, 2.0, 1.25))
    out, s = oracle.recurrence_forward(k, k, np.ones(3, np.float32), np.zeros(3, np.float32), st)
    assert out.shape == (2, 0, 3)
    assert np.allclose(s[0], 0.5) and np.allclose(s[1], 2.0) and np.allclose(s[2], 1.25)


# ---------------------------------------------------------------------------
# planted mistakes: a Python copy of the recurrence with one thing broken must
# fail at least one check
# ---------------------------------------------------------------------------

def _python_recurrence(mistake=None):
    def impl(k, v, w, u, st):
        k = np.asarray(k, np.float64)
        v = np.asarray(v, np.float64)
        B, T, C = k.shape
        out = np.empty((B, T, C))
        if st is None:
            num, den, m = np.zeros((B, C)), np.zeros((B, C)), np.full((B, C), -np.inf)
        else:
            num, den, m = (np.array(x, np.float64) for x in st)
        wd = np.asarray(w, np.float64)
        ud = np.asarray(u, np.float64)
        if mistake == "decay_sign":
            wd = -wd
        if mistake == "no_bonus":
            ud = 0.0 * ud
        with np.errstate(invalid="ignore"):
            for t in range(T):
                kt, vt = k[:, t], v[:, t]
                if mistake == "decay_before_output":
                    m = m - wd
                kb = kt + ud
                e = np.maximum(m, kb)
                a, b = np.exp(m - e), np.exp(kb - e)
                if mistake == "swap_num_den":
                    out[:, t] = (a * den + b * vt) / (a * num + b)
                elif mistake == "drop_current":
                    out[:, t] = (a * num + 0 * b * vt) / (a * den + b)
                else:
                    out[:, t] = (a * num + b * vt) / (a * den + b)
                md = m if mistake == "decay_before_output" else m - wd
                if mistake == "bonus_in_state":
                    kt = kt + ud
                if mistake == "double_decay":
                    md = md - wd
                e2 = np.maximum(md, kt)
                a2, b2 = np.exp(md - e2), np.exp(kt - e2)
                num = a2 * num + b2 * vt
                den = a2 * den + b2
                m = e2
        return out, (num, den, m)
    return impl


def test_python_recurrence_passes():
    for check in ALL_CHECKS:
        check(_python_recurrence())


@pytest.mark.parametrize("mistake", ["decay_sign", "no_bonus", "decay_before_output",
                                     "swap_num_den", "drop_current", "bonus_in_state",
                                     "double_decay"])
def test_pins_catch_planted_mistakes(mistake):
    impl = _python_recurrence(mistake)
    failed = []
    for check in ALL_CHECKS:
        try:
            check(impl)
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"no check caught the planted mistake {mistake!r}"


# ---------------------------------------------------------------------------
# the two extensions of "RWKV-v6 Architecture: Attention-Free Linear
# Transformers": per-token decay w_t (section "2. Dynamic Data-Dependent
# Decay") and the receptance gate sigmoid(r) * wkv. Checks take
# impl(k, v, w, u, state, w_t, r) -> (out, state).
# ---------------------------------------------------------------------------

GOLDEN_EXT = os.path.join(os.path.dirname(__file__), "golden", "wkv_tiny_wt_gate_decimal.txt")


def load_golden_ext():
    rows = [ln.split() for ln in open(GOLDEN_EXT) if not ln.startswith("#")]
    B = 1 + max(int(r[0]) for r in rows)
    T = 1 + max(int(r[1]) for r in rows)
    C = 1 + max(int(r[2]) for r in rows)
    k, v, wt, r_ = (np.zeros((B, T, C), np.float32) for _ in range(4))
    w = np.zeros(C, np.float32)
    u = np.zeros(C, np.float32)
    ref = np.zeros((B, T, C))
    for row in rows:
        b, t, c = int(row[0]), int(row[1]), int(row[2])
        k[b, t, c], v[b, t, c], wt[b, t, c], u[c], r_[b, t, c] = (np.float32(float(x)) for x in row[3:8])
        ref[b, t, c] = float(row[8])
    return k, v, w, u, wt, r_, ref


def check_ext_hand_worked(impl):
    """Three tokens, one channel, worked by hand, with per-token decays
    w_t = (ln 2, ln 3, ln 5), k = 0, v = (1, 2, 4), u = 0 and no gate.

    Token 1 sees only itself: 1. Token 2 sees token 1 undecayed and itself:
    (1 + 2) / 2 = 3/2. Token 2's advance decays the state by e^{-ln 3}: the
    pair becomes N = 1/3 + 2, D = 1/3 + 1, so token 3 gives (7/3 + 4) / (4/3 + 1)
    = 19/7. Token 3's advance decays by 1/5: N = 67/15, D = 19/15 over the
    largest exponent 0 (token 3's key).
    """
    k = np.zeros((1, 3, 1), np.float32)
    v = np.array([1.0, 2.0, 4.0], np.float32).reshape(1, 3, 1)
    wt = np.log(np.array([2.0, 3.0, 5.0])).astype(np.float32).reshape(1, 3, 1)
    out, (num, den, mx) = impl(k, v, np.zeros(1, np.float32), np.zeros(1, np.float32), None, wt, None)
    assert out[0, :, 0] == pytest.approx([1.0, 1.5, 19.0 / 7.0], rel=1e-6)
    assert num[0, 0] == pytest.approx(67.0 / 15.0, rel=1e-6)
    assert den[0, 0] == pytest.approx(19.0 / 15.0, rel=1e-6)
    assert mx[0, 0] == pytest.approx(0.0, abs=1e-7)


def check_ext_golden_decimal(impl, tol=1e-12):
    k, v, w, u, wt, r, ref = load_golden_ext()
    out, _ = impl(k, v, w, u, None, wt, r)
    assert np.abs(out - ref).max() <= tol * max(1.0, np.abs(ref).max())


def check_ext_constant_decay_reduces(impl):
    """w_t equal to w at every token is the per-channel equation (whose pins
    are above): compared with the hand-worked and golden-pinned recurrence."""
    from oracle import oracle as O
    k, v, w, u, st = I.random_case(2, 40, 6, 31, k_scale=2.0, k_spike=30.0, state=True)
    wt = np.broadcast_to(w, k.shape).copy()
    out, s = impl(k, v, w, u, st, wt, None)
    ref, rs = O.recurrence_forward(k, v, w, u, st)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-13)
    assert np.allclose(s[2] + np.log(s[1]), rs[2] + np.log(rs[1]), rtol=0, atol=1e-12)


def check_ext_reset(impl):
    """A decay of 1e4 at token j erases every earlier token from the outputs
    after j: they equal a run that starts at token j from the empty state."""
    k, v, w, u, _ = I.random_case(1, 30, 5, 32, k_scale=2.0)
    g = np.random.default_rng(32)
    wt = np.exp(g.normal(-1.0, 1.0, k.shape)).astype(np.float32)
    j = 11
    wt[:, j] = np.float32(1e4)
    out, _ = impl(k, v, w, u, None, wt, None)
    out_j, _ = impl(k[:, j:], v[:, j:], w, u, None, wt[:, j:], None)
    assert np.allclose(out[:, j + 1:], out_j[:, 1:], rtol=1e-12, atol=1e-14)
    assert not np.allclose(out[:, j], out_j[:, 0])  # token j itself still sees the past


def check_ext_split(impl):
    """Per-token decays and the gate: T1 tokens then the rest from the state = one pass."""
    k, v, w, u, st = I.random_case(2, 41, 5, 33, k_scale=2.0, state=True)
    g = np.random.default_rng(33)
    wt = np.exp(g.normal(-2.0, 1.5, k.shape)).astype(np.float32)
    r = g.normal(0.0, 2.0, k.shape).astype(np.float32)
    out, s = impl(k, v, w, u, st, wt, r)
    o1, s1 = impl(k[:, :13], v[:, :13], w, u, st, wt[:, :13], r[:, :13])
    o2, s2 = impl(k[:, 13:], v[:, 13:], w, u, s1, wt[:, 13:], r[:, 13:])
    assert np.allclose(np.concatenate([o1, o2], 1), out, rtol=1e-12, atol=1e-13)
    assert np.allclose(s2[2] + np.log(s2[1]), s[2] + np.log(s[1]), rtol=0, atol=1e-12)


def check_gate_values(impl):
    """r = 0 halves every output exactly (sigmoid(0) = 1/2) and leaves the state
    alone; r = +40 leaves it (to 1e-17); r = -40 sends it to zero (e^-40)."""
    k, v, w, u, st = I.random_case(2, 25, 4, 34, k_scale=2.0, state=True)
    plain, s0 = impl(k, v, w, u, st, None, None)
    half, s1 = impl(k, v, w, u, st, None, np.zeros_like(k))
    assert np.array_equal(half, plain * 0.5)
    for a, b in zip(s0, s1):
        assert np.array_equal(a, b)
    hi, _ = impl(k, v, w, u, st, None, np.full_like(k, 40.0))
    assert np.allclose(hi, plain, rtol=1e-16, atol=0)
    lo, _ = impl(k, v, w, u, st, None, np.full_like(k, -40.0))
    assert np.all(np.abs(lo) <= 5e-18 * np.abs(plain) + 1e-300)


EXT_CHECKS = [check_ext_hand_worked, check_ext_golden_decimal, check_ext_constant_decay_reduces,
              check_ext_reset, check_ext_split, check_gate_values]


def _recurrence_ext(O):
    return lambda k, v, w, u, st, wt, r: O.recurrence_forward(k, v, w, u, st, w_t=wt, r=r)


def _direct_ext(O):
    return lambda k, v, w, u, st, wt, r: O.direct_forward(k, v, w, u, st, w_t=wt, r=r)


@pytest.mark.parametrize("check", EXT_CHECKS, ids=lambda f: f.__name__)
def test_recurrence_ext_pins(oracle, check):
    check(_recurrence_ext(oracle))


@pytest.mark.parametrize("check", EXT_CHECKS, ids=lambda f: f.__name__)
def test_direct_sum_ext_pins(oracle, check):
    check(_direct_ext(oracle))


def test_decimal_ext_matches_golden(oracle):
    k, v, w, u, wt, r, ref = load_golden_ext()
    res = oracle.decimal_forward(k, v, w, u, digits=50, w_t=wt, r=r)
    for (b, t, c), x in np.ndenumerate(ref):
        assert abs(float(res[b][t][c]) - x) <= 1e-15 * max(1.0, abs(x))


@pytest.mark.parametrize("seed", range(4))
def test_recurrence_ext_equals_direct_sum(oracle, seed):
    T = [9, 33, 64, 50][seed]
    k, v, w, u, st = I.random_case(2, T, 7, 200 + seed, k_scale=1.0 + seed, k_spike=[0, 40, 0, 60][seed],
                                   state=bool(seed % 2))
    g = np.random.default_rng(200 + seed)
    wt = np.exp(g.normal(-1.0 - seed, 1.5, k.shape)).astype(np.float32)
    r = g.normal(0.0, 2.0, k.shape).astype(np.float32) if seed % 2 == 0 else None
    o1, s1 = oracle.recurrence_forward(k, v, w, u, st, w_t=wt, r=r)
    o2, s2 = oracle.direct_forward(k, v, w, u, st, w_t=wt, r=r)
    scale, _ = oracle.abs_scale_forward(k, v, w, u, st, w_t=wt, r=r)
    assert np.all(np.abs(o1 - o2) <= 1e-12 * scale + 1e-300)
    assert np.allclose(s1[2] + np.log(s1[1]), s2[2] + np.log(s2[1]), rtol=0, atol=1e-12)
    assert np.allclose(s1[0] / s1[1], s2[0] / s2[1], rtol=1e-12, atol=1e-13)
    assert np.all(np.abs(o1) <= scale * (1 + 1e-12))


def test_ext_direct_output_and_step(oracle):
    """direct_output and recurrence_step (per-stream decay, gate) against the forward."""
    k, v, w, u, st = I.random_case(2, 20, 3, 35, state=True)
    g = np.random.default_rng(35)
    wt = np.exp(g.normal(-1.0, 1.0, k.shape)).astype(np.float32)
    r = g.normal(0.0, 1.0, k.shape).astype(np.float32)
    out, s = oracle.recurrence_forward(k, v, w, u, st, w_t=wt, r=r)
    for t in (0, 1, 19):
        o = oracle.direct_output(k[1, :, 2], v[1, :, 2], w[2], u[2], t, (st[0][1, 2], st[1][1, 2], st[2][1, 2]),
                                 w_t=wt[1, :, 2], r=r[1, t, 2])
        assert o == pytest.approx(out[1, t, 2], rel=1e-13, abs=1e-15)
    state = tuple(x.astype(np.float64) for x in st)
    for t in range(k.shape[1]):
        o, state = oracle.recurrence_step(state, k[:, t], v[:, t], wt[:, t], u, r=r[:, t])
        assert np.array_equal(o, out[:, t])
    for a, b in zip(state, s):
        assert np.array_equal(a, b)


def _python_recurrence_ext(mistake=None):
    """A Python copy of the recurrence with w_t and the gate, and one thing broken."""
    def impl(k, v, w, u, st, wt, r):
        k = np.asarray(k, np.float64)
        v = np.asarray(v, np.float64)
        B, T, C = k.shape
        wt = np.broadcast_to(np.asarray(w, np.float64), k.shape) if wt is None else np.asarray(wt, np.float64)
        out = np.empty((B, T, C))
        if st is None:
            num, den, m = np.zeros((B, C)), np.zeros((B, C)), np.full((B, C), -np.inf)
        else:
            num, den, m = (np.array(x, np.float64) for x in st)
        ud = np.asarray(u, np.float64)
        with np.errstate(invalid="ignore"):
            for t in range(T):
                kt, vt = k[:, t], v[:, t]
                kb = kt + ud
                e = np.maximum(m, kb)
                a, b = np.exp(m - e), np.exp(kb - e)
                y = (a * num + b * vt) / (a * den + b)
                if r is not None:
                    rr = np.asarray(r, np.float64)[:, t]
                    y = y / (1 + np.exp(rr if mistake == "gate_sign" else -rr))
                out[:, t] = y
                if mistake == "decay_next_token":
                    wd = wt[:, min(t + 1, T - 1)]
                elif mistake == "decay_prev_token":
                    wd = wt[:, max(t - 1, 0)]
                else:
                    wd = wt[:, t]
                md = m - wd
                e2 = np.maximum(md, kt)
                a2, b2 = np.exp(md - e2), np.exp(kt - e2)
                num = a2 * num + b2 * vt
                den = a2 * den + b2
                m = e2
        return out, (num, den, m)
    return impl


def test_python_recurrence_ext_passes():
    for check in EXT_CHECKS:
        check(_python_recurrence_ext())


@pytest.mark.parametrize("mistake", ["decay_next_token", "decay_prev_token", "gate_sign"])
def test_ext_pins_catch_planted_mistakes(mistake):
    impl = _python_recurrence_ext(mistake)
    failed = []
    for check in EXT_CHECKS:
        try:
            check(impl)
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"no check caught the planted mistake {mistake!r}"
