"""Pins for the oracle's backward (no GPU).

recurrence_backward returns the gradients of L = sum_t g_t * wkv_t with
respect to k, v, w, u and the state passed in, by the chain rule run backwards
through the step function of "Linear attention without writing a CUDA
kernel", section "The recurrence". It is tied here to things other than
itself:

* central finite differences of the direct sum of the wkv_t equation (numpy,
  float64) -- the definition, differentiated numerically;
* torch autograd (float64, CPU) of the equation restated as a causal softmax
  whose scores are k_i - (t-1-i) w, u + k_t on the diagonal, and the state as
  one more column with score m0 + ln den0 - t w and value num0 / den0;
* invariants that hold for any inputs: shifting every v and the state's
  num0 / den0 by the same amount shifts every output by it, so
  sum_t dv_t + den0 dnum0 = sum_t g_t; shifting every key and m0 by the same
  amount changes nothing, so sum_t dk_t + dm0 = 0;
* the scales it returns bound the gradients (|grad| <= scale);
* deliberately broken copies of the backward fail at least one check.
"""
import math

import numpy as np
import pytest
import torch

from wkv_recurrence_b200 import inputs as I


def _case(seed, B=2, T=9, C=3, spike=0.0, state=True, w_range=(1e-3, 8.0)):
    k, v, w, u, st = I.random_case(B, T, C, seed=seed, k_scale=1.5, k_spike=spike, w_range=w_range, state=state)
    g = np.random.default_rng(seed + 1000).normal(size=k.shape)
    if st is not None:
        st = tuple(x.astype(np.float64) for x in st)
    return k, v, w, u, st, g


def _loss(O, k, v, w, u, st, g):
    out, _ = O.direct_forward(k, v, w, u, st)
    return float((out * g).sum())


def _fd(O, k, v, w, u, st, g, which, idx, h=1e-6):
    """Central difference of the direct-sum loss in one input element."""
    args = {"k": k.astype(np.float64), "v": v.astype(np.float64), "w": w.astype(np.float64),
            "u": u.astype(np.float64)}
    sts = None if st is None else [x.copy() for x in st]
    vals = []
    for sgn in (1.0, -1.0):
        a = {n: x.copy() for n, x in args.items()}
        s = None if sts is None else [x.copy() for x in sts]
        if which in a:
            a[which][idx] += sgn * h
        else:
            s[{"dnum": 0, "dden": 1, "dmax": 2}[which]][idx] += sgn * h
        vals.append(_loss(O, a["k"], a["v"], a["w"], a["u"], None if s is None else tuple(s), g))
    return (vals[0] - vals[1]) / (2 * h)


GRADS = {"dk": "k", "dv": "v", "dw": "w", "du": "u"}


def check_finite_differences(bwd, O):
    for seed, spike, state in ((1, 0.0, True), (2, 20.0, True), (3, 0.0, False)):
        k, v, w, u, st, g = _case(seed, spike=spike, state=state)
        d, _ = bwd(k, v, w, u, g, st)
        rng = np.random.default_rng(seed)
        for name, which in GRADS.items():
            shape = d[name].shape
            for _ in range(4):
                idx = tuple(int(rng.integers(n)) for n in shape)
                ref = _fd(O, k, v, w, u, st, g, which, idx)
                assert d[name][idx] == pytest.approx(ref, rel=1e-6, abs=1e-8), (name, idx, seed)
        if state:
            for name in ("dnum", "dden", "dmax"):
                idx = (1, 2)
                ref = _fd(O, k, v, w, u, st, g, name, idx)
                assert d[name][idx] == pytest.approx(ref, rel=1e-6, abs=1e-8), (name, seed)


def _torch_grads(k, v, w, u, st, g):
    """Autograd of the causal-softmax restatement, float64."""
    B, T, C = k.shape
    K = torch.tensor(k, dtype=torch.float64, requires_grad=True)
    V = torch.tensor(v, dtype=torch.float64, requires_grad=True)
    Wt = torch.tensor(w, dtype=torch.float64, requires_grad=True)
    U = torch.tensor(u, dtype=torch.float64, requires_grad=True)
    S = [torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in st]
    t = torch.arange(T, dtype=torch.float64)
    # scores[b, c, t, i] for the tokens; column -1 for the state
    kk = K.permute(0, 2, 1)  # [B, C, T]
    dist = (t[:, None] - 1 - t[None, :])  # t-1-i
    sc = kk[:, :, None, :] - dist[None, None] * Wt[None, :, None, None]
    diag = torch.eye(T, dtype=torch.bool)
    sc = torch.where(diag, (U[None, :, None] + kk)[:, :, :, None].expand(B, C, T, T), sc)
    sc = sc.masked_fill(torch.triu(torch.ones(T, T, dtype=torch.bool), 1), -math.inf)
    st_score = (S[2] + torch.log(S[1]))[:, :, None] - t[None, None, :] * Wt[None, :, None]
    allsc = torch.cat([sc, st_score[..., None]], dim=-1)
    vals = torch.cat([V.permute(0, 2, 1)[:, :, None, :].expand(B, C, T, T),
                      (S[0] / S[1])[:, :, None, None].expand(B, C, T, 1)], dim=-1)
    out = (torch.softmax(allsc, dim=-1) * vals).sum(-1)  # [B, C, T]
    loss = (out.permute(0, 2, 1) * torch.tensor(g)).sum()
    loss.backward()
    return {"dk": K.grad.numpy(), "dv": V.grad.numpy(), "dw": Wt.grad.numpy(), "du": U.grad.numpy(),
            "dnum": S[0].grad.numpy(), "dden": S[1].grad.numpy(), "dmax": S[2].grad.numpy()}


def check_autograd(bwd, O):
    for seed, spike in ((11, 0.0), (12, 30.0), (13, 0.0)):
        k, v, w, u, st, g = _case(seed, B=2, T=24, C=4, spike=spike, w_range=(1e-3, 4.0))
        d, _ = bwd(k, v, w, u, g, st)
        ref = _torch_grads(k, v, w, u, st, g)
        for name in ("dk", "dv", "dw", "du", "dnum", "dden", "dmax"):
            scale = np.abs(ref[name]).max() + 1e-300
            assert np.abs(d[name] - ref[name]).max() <= 1e-11 * scale, (name, seed)


def check_shift_invariants(bwd, O):
    k, v, w, u, st, g = _case(21, B=3, T=30, C=5, spike=15.0)
    d, _ = bwd(k, v, w, u, g, st)
    lhs = d["dv"].sum(axis=1) + st[1] * d["dnum"]
    assert np.allclose(lhs, g.sum(axis=1), rtol=1e-11, atol=1e-11)
    assert np.allclose(d["dk"].sum(axis=1) + d["dmax"], 0.0, atol=1e-11 * np.abs(d["dk"]).sum(axis=1).max())
    # without a state: sum_t dv_t = sum_t g_t and sum_t dk_t = 0
    k, v, w, u, _, g = _case(22, B=2, T=17, C=4, state=False)
    d, _ = bwd(k, v, w, u, g, None)
    assert np.allclose(d["dv"].sum(axis=1), g.sum(axis=1), rtol=1e-11, atol=1e-11)
    assert np.allclose(d["dk"].sum(axis=1), 0.0, atol=1e-11 * max(1.0, np.abs(d["dk"]).sum(axis=1).max()))


ALL = [check_finite_differences, check_autograd, check_shift_invariants]


@pytest.mark.parametrize("check", ALL, ids=lambda f: f.__name__)
def test_backward_pins(oracle, check):
    check(lambda k, v, w, u, g, st: oracle.recurrence_backward(k, v, w, u, g, st), oracle)


def test_backward_scales_bound_the_gradients(oracle):
    for seed in range(3):
        k, v, w, u, st, g = _case(30 + seed, B=2, T=40, C=6, spike=[0.0, 40.0, 100.0][seed])
        d, sc = oracle.recurrence_backward(k, v, w, u, g, st)
        for name in d:
            assert np.all(np.abs(d[name]) <= sc[name] * (1 + 1e-12) + 1e-300), name
            assert np.all(np.isfinite(d[name])) and np.all(np.isfinite(sc[name])), name


def test_backward_bf16_inputs_widen_exactly(oracle):
    k, v, w, u, st, g = _case(40, B=2, T=20, C=3)
    kb, vb = I.f32_to_bf16_bits(k), I.f32_to_bf16_bits(v)
    d1, _ = oracle.recurrence_backward(kb, vb, w, u, g, st, kv_dtype="bf16")
    d2, _ = oracle.recurrence_backward(I.bf16_bits_to_f32(kb), I.bf16_bits_to_f32(vb), w, u, g, st)
    for name in d1:
        assert np.array_equal(d1[name], d2[name]), name


def test_backward_of_empty_sequence(oracle):
    k = np.zeros((2, 0, 3), np.float32)
    st = tuple(np.full((2, 3), x) for x in (0.5, 2.0, 1.25))
    d, _ = oracle.recurrence_backward(k, k, np.ones(3, np.float32), np.zeros(3, np.float32), np.zeros((2, 0, 3)), st)
    for name in d:
        assert np.all(d[name] == 0), name


# ---------------------------------------------------------------------------
# planted mistakes: a Python copy of the backward with one thing broken must
# fail at least one check
# ---------------------------------------------------------------------------

def _python_backward(mistake=None):
    def bwd(k, v, w, u, g, st):
        k = np.asarray(k, np.float64)
        v = np.asarray(v, np.float64)
        B, T, C = k.shape
        d = {"dk": np.zeros((B, T, C)), "dv": np.zeros((B, T, C)), "dw": np.zeros(C), "du": np.zeros(C),
             "dnum": np.zeros((B, C)), "dden": np.zeros((B, C)), "dmax": np.zeros((B, C))}
        for b in range(B):
            for c in range(C):
                wc, uc = float(w[c]), float(u[c])
                if st is None:
                    num, den, m = 0.0, 0.0, -math.inf
                else:
                    num, den, m = (float(x[b, c]) for x in st)
                num0, den0, m0 = num, den, m
                states = []
                for t in range(T):
                    states.append((num, den, m))
                    kt, vt = k[b, t, c], v[b, t, c]
                    md = m - wc
                    e2 = max(md, kt)
                    a2, b2 = math.exp(md - e2), math.exp(kt - e2)
                    num, den, m = a2 * num + b2 * vt, a2 * den + b2, e2
                rn = rd = 0.0
                Q = -math.inf
                for t in range(T - 1, -1, -1):
                    kt, vt, gt = k[b, t, c], v[b, t, c], g[b, t, c]
                    nt, dt, mt = states[t]
                    e = max(mt, kt + uc)
                    a, bb = math.exp(mt - e), math.exp(kt + uc - e)
                    z = a * dt + bb
                    out = (a * nt + bb * vt) / z
                    p, q = gt / z, -gt * out / z
                    if mistake == "q_sign":
                        q = -q
                    E1 = math.exp(kt + Q)
                    E2 = math.exp(mt + Q - (0.0 if mistake == "dw_no_decay" else wc))
                    d["dv"][b, t, c] = (0.0 if mistake == "dv_no_local" else p * bb) + rn * E1
                    d["dk"][b, t, c] = p * bb * (vt - out) + E1 * (vt * rn + (0.0 if mistake == "dk_no_den" else rd))
                    d["du"][c] += p * bb * (vt - out)
                    d["dw"][c] -= E2 * (nt * rn + dt * rd)
                    decay = 0.0 if mistake == "reverse_no_decay" else wc
                    Qn = max(Q - decay, -e)
                    x1, x2 = math.exp(Q - decay - Qn), math.exp(-e - Qn)
                    rn, rd, Q = rn * x1 + p * x2, rd * x1 + q * x2, Qn
                if st is not None and m0 > -math.inf:
                    f = math.exp(m0 + Q)
                    d["dnum"][b, c], d["dden"][b, c] = rn * f, rd * f
                    d["dmax"][b, c] = num0 * rn * f + den0 * rd * f
        return d, None
    return bwd


def test_python_backward_passes(oracle):
    for check in ALL:
        check(_python_backward(), oracle)


@pytest.mark.parametrize("mistake", ["q_sign", "dw_no_decay", "dv_no_local", "dk_no_den", "reverse_no_decay"])
def test_backward_pins_catch_planted_mistakes(oracle, mistake):
    failed = []
    for check in ALL:
        try:
            check(_python_backward(mistake), oracle)
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"no check caught the planted mistake {mistake!r}"
