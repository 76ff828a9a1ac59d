"""Pins for the RWKV-v6 matrix-state oracle (no GPU).

"RWKV-v6 Architecture: Attention-Free Linear Transformers", section
"3. Matrix-Valued Hidden State": S_t = diag(w_t) S_{t-1} + k_t v_t^T and
y_t = sigmoid(r_t) * (S_t k_t). The oracle's recurrence is tied to the closed
form (the sum written out), to hand-worked examples that fix which index
decays and which one the readout contracts, to a library matrix-product
restatement when nothing decays (w = 1), to closed forms for w = 0 and r = 0,
and to planted mistakes that must fail.
"""
import math

import numpy as np
import pytest
import torch

from oracle import v6_oracle as V


def _case(seed, B=2, T=7, H=2, D=4, state=True):
    g = np.random.default_rng(seed)
    r = g.normal(0, 1, (B, T, H, D)).astype(np.float32)
    w = np.exp(-np.exp(g.normal(-1, 1, (B, T, H, D)))).astype(np.float32)
    k = g.normal(0, 1, (B, T, H, D)).astype(np.float32)
    v = g.normal(0, 1, (B, T, H, D)).astype(np.float32)
    s = g.normal(0, 1, (B, H, D, D)) if state else None
    return r, w, k, v, s


def check_hand_worked_scalar(impl):
    """D = 1: S_1 = 0.5*0 + 1*3 = 3, y_1 = sigmoid(0)*3*1 = 1.5;
    S_2 = 0.25*3 + 2*4 = 8.75, y_2 = 0.5*8.75*2 = 8.75."""
    r = np.zeros((1, 2, 1, 1), np.float32)
    w = np.array([0.5, 0.25], np.float32).reshape(1, 2, 1, 1)
    k = np.array([1.0, 2.0], np.float32).reshape(1, 2, 1, 1)
    v = np.array([3.0, 4.0], np.float32).reshape(1, 2, 1, 1)
    y, S = impl(r, w, k, v, None)
    assert y[0, :, 0, 0] == pytest.approx([1.5, 8.75], rel=1e-15)
    assert S[0, 0, 0, 0] == pytest.approx(8.75, rel=1e-15)


def check_hand_worked_matrix(impl):
    """D = 2, one token, S_0 = [[1, 2], [3, 4]], w = (0.5, 0.25), k = (1, 2),
    v = (3, -1), gate open (r = 40): row i decays by w[i] and gains k[i] v^T:
    S_1 = [[0.5 + 3, 1 - 1], [0.75 + 6, 1 - 2]] = [[3.5, 0], [6.75, -1]], and the
    readout contracts the column index with k: y = S_1 k = (3.5, 4.75)."""
    S0 = np.array([[[[1.0, 2.0], [3.0, 4.0]]]])
    r = np.full((1, 1, 1, 2), 40.0, np.float32)
    w = np.array([0.5, 0.25], np.float32).reshape(1, 1, 1, 2)
    k = np.array([1.0, 2.0], np.float32).reshape(1, 1, 1, 2)
    v = np.array([3.0, -1.0], np.float32).reshape(1, 1, 1, 2)
    y, S = impl(r, w, k, v, S0)
    assert np.allclose(S[0, 0], [[3.5, 0.0], [6.75, -1.0]], rtol=1e-15, atol=0)
    assert np.allclose(y[0, 0, 0], [3.5, 4.75], rtol=1e-15)


def check_no_decay_is_a_masked_matmul(impl):
    """w = 1 (nothing fades): y_t = sigmoid(r_t) * sum_{s<=t} k_s (v_s . k_t),
    i.e. Y = sigmoid(R) * (tril(K V^T) K) per head (torch matmul)."""
    r, w, k, v, _ = _case(3, T=9, state=False)
    w[:] = 1.0
    y, _ = impl(r, w, k, v, None)
    B, T, H, D = k.shape
    for b in range(B):
        for h in range(H):
            K = torch.tensor(k[b, :, h], dtype=torch.float64)
            Vv = torch.tensor(v[b, :, h], dtype=torch.float64)
            M = torch.tril(K @ Vv.T)
            ref = torch.sigmoid(torch.tensor(r[b, :, h], dtype=torch.float64)) * (M @ K)
            assert np.allclose(y[b, :, h], ref.numpy(), rtol=1e-12, atol=1e-12)


def check_full_decay(impl):
    """w = 0: only the current token survives: y_t = sigmoid(r_t) k_t (v_t . k_t)."""
    r, w, k, v, s = _case(4)
    w[:] = 0.0
    y, _ = impl(r, w, k, v, s)
    kd, vd, rd = (x.astype(np.float64) for x in (k, v, r))
    ref = (1 / (1 + np.exp(-rd))) * kd * (vd * kd).sum(-1, keepdims=True)
    assert np.allclose(y, ref, rtol=1e-13, atol=1e-13)


def check_gate_half(impl):
    r, w, k, v, s = _case(5)
    y1, _ = impl(np.zeros_like(r), w, k, v, s)
    y2, _ = impl(np.full_like(r, 40.0), w, k, v, s)
    assert np.allclose(y1, 0.5 * y2, rtol=1e-14, atol=1e-14)


def check_split(impl):
    r, w, k, v, s = _case(6, T=11)
    y, S = impl(r, w, k, v, s)
    y1, S1 = impl(r[:, :4], w[:, :4], k[:, :4], v[:, :4], s)
    y2, S2 = impl(r[:, 4:], w[:, 4:], k[:, 4:], v[:, 4:], S1)
    assert np.allclose(np.concatenate([y1, y2], 1), y, rtol=1e-12, atol=1e-12)
    assert np.allclose(S2, S, rtol=1e-12, atol=1e-12)


CHECKS = [check_hand_worked_scalar, check_hand_worked_matrix, check_no_decay_is_a_masked_matmul,
          check_full_decay, check_gate_half, check_split]


@pytest.mark.parametrize("check", CHECKS, ids=lambda f: f.__name__)
@pytest.mark.parametrize("form", ["recurrence", "direct"])
def test_v6_pins(check, form):
    check(getattr(V, form))


@pytest.mark.parametrize("seed", range(4))
def test_v6_recurrence_equals_direct(seed):
    r, w, k, v, s = _case(10 + seed, T=[1, 6, 13, 20][seed], D=[1, 4, 8, 3][seed], state=bool(seed % 2))
    y1, S1 = V.recurrence(r, w, k, v, s)
    y2, S2 = V.direct(r, w, k, v, s)
    sc, _ = V.abs_scale(r, w, k, v, s)
    assert np.all(np.abs(y1 - y2) <= 1e-12 * sc + 1e-300)
    assert np.allclose(S1, S2, rtol=1e-12, atol=1e-12)
    assert np.all(np.abs(y1) <= sc * (1 + 1e-12))


def test_v6_bf16_widens_exactly():
    from wkv_recurrence_b200 import inputs as I
    r, w, k, v, s = _case(20)
    rb, kb, vb = (I.f32_to_bf16_bits(x) for x in (r, k, v))
    y1, _ = V.recurrence(rb, w, kb, vb, s, kv_dtype="bf16")
    y2, _ = V.recurrence(*(I.bf16_bits_to_f32(x) for x in (rb,)), w, I.bf16_bits_to_f32(kb),
                         I.bf16_bits_to_f32(vb), s)
    assert np.array_equal(y1, y2)


def _python_v6(mistake=None):
    def impl(r, w, k, v, state):
        r, w, k, v = (np.asarray(x, np.float64) for x in (r, w, k, v))
        B, T, H, D = k.shape
        S = np.zeros((B, H, D, D)) if state is None else np.array(state, np.float64)
        y = np.empty((B, T, H, D))
        for t in range(T):
            Sp = S
            if mistake == "column_decay":
                S = w[:, t, :, None, :] * S + k[:, t, :, :, None] * v[:, t, :, None, :]
            elif mistake == "outer_swapped":
                S = w[:, t, :, :, None] * S + v[:, t, :, :, None] * k[:, t, :, None, :]
            else:
                S = w[:, t, :, :, None] * S + k[:, t, :, :, None] * v[:, t, :, None, :]
            Sr = Sp if mistake == "read_old_state" else S
            if mistake == "transposed_readout":
                o = np.einsum("bhji,bhj->bhi", Sr, k[:, t])
            else:
                o = np.einsum("bhij,bhj->bhi", Sr, k[:, t])
            gate = 1 / (1 + np.exp(r[:, t] if mistake == "gate_sign" else -r[:, t]))
            y[:, t] = gate * o
        return y, S
    return impl


def test_python_v6_passes():
    for check in CHECKS:
        check(_python_v6())


@pytest.mark.parametrize("mistake", ["column_decay", "outer_swapped", "read_old_state", "transposed_readout",
                                     "gate_sign"])
def test_v6_pins_catch_planted_mistakes(mistake):
    failed = []
    for check in CHECKS:
        try:
            check(_python_v6(mistake))
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"no check caught the planted mistake {mistake!r}"
