"""CPU oracle for the RWKV-v6 matrix-valued state (float64).

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the product path; it shares no code
with the CUDA library.

Source: "RWKV-v6 Architecture: Attention-Free Linear Transformers", section
"3. Matrix-Valued Hidden State" and the readout under it. Per head the state
is a d x d matrix S and every token (r_t, w_t, k_t, v_t), each a d-vector,
updates and reads it:

    S_t = diag(w_t) S_{t-1} + k_t v_t^T          (row i decays by w_t[i])
    y_t = sigmoid(r_t) * (S_t k_t)               (elementwise gate)

w_t is the decay factor itself (the page forms it as exp(-exp(.)) of a
projection; here it is an input in (0, 1]). Note that the readout multiplies
the updated state S_t by k_t, as the page's equation and its module both
write it.

Layout: r, w, k, v, y are [B, T, H, D]; the state is [B, H, D, D] with
S[b, h, i, j] the entry of row i (key dimension) and column j (value
dimension).

Functions
---------
``recurrence``     the two lines above, token by token (numpy float64).
``direct``         the closed form of the same thing, the sum written out:
                   S_t = sum_{s<=t} P(s,t) k_s v_s^T + P(0,t) S_0 with
                   P(s,t) = diag(w_{s+1} ... w_t), so
                   y_t[i] = sigmoid(r_t[i]) (sum_{s<=t} P(s,t)[i] k_s[i] (v_s . k_t)
                                             + P(0,t)[i] (S_0 k_t)[i]).
                   O(T^2): small cases.
``abs_scale``      the recurrence on magnitudes (|k|, |v|, |S_0|, and |k_t| in
                   the readout): the per-output scale sum of |terms| against
                   which rounding error is measured.
Parity unpinned: none (pins in tests/test_v6_oracle.py).
"""
from __future__ import annotations

import numpy as np


def _f64(x, dtype="f32"):
    if dtype == "bf16":
        return (np.asarray(x, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return np.asarray(x, np.float64)


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def recurrence(r, w, k, v, state=None, kv_dtype: str = "f32"):
    """Token-by-token float64. Returns (y [B, T, H, D], S_T [B, H, D, D])."""
    r, k, v = _f64(r, kv_dtype), _f64(k, kv_dtype), _f64(v, kv_dtype)
    w = np.asarray(w, np.float64)
    B, T, H, D = k.shape
    S = np.zeros((B, H, D, D)) if state is None else np.array(state, np.float64)
    y = np.empty((B, T, H, D))
    for t in range(T):
        S = w[:, t, :, :, None] * S + k[:, t, :, :, None] * v[:, t, :, None, :]
        y[:, t] = _sigmoid(r[:, t]) * np.einsum("bhij,bhj->bhi", S, k[:, t])
    return y, S


def direct(r, w, k, v, state=None, kv_dtype: str = "f32"):
    """The closed form (sum over earlier tokens with products of decays)."""
    r, k, v = _f64(r, kv_dtype), _f64(k, kv_dtype), _f64(v, kv_dtype)
    w = np.asarray(w, np.float64)
    B, T, H, D = k.shape
    S0 = np.zeros((B, H, D, D)) if state is None else np.array(state, np.float64)
    y = np.empty((B, T, H, D))
    for t in range(T):
        acc = np.zeros((B, H, D))
        for s in range(t + 1):
            P = np.prod(w[:, s + 1:t + 1], axis=1)              # [B, H, D]: decays of tokens s+1..t
            dot = np.einsum("bhj,bhj->bh", v[:, s], k[:, t])     # v_s . k_t
            acc += P * k[:, s] * dot[..., None]
        P0 = np.prod(w[:, :t + 1], axis=1)
        acc += P0 * np.einsum("bhij,bhj->bhi", S0, k[:, t])
        y[:, t] = _sigmoid(r[:, t]) * acc
    ST = np.prod(w, axis=1)[..., None] * S0
    for s in range(T):
        P = np.prod(w[:, s + 1:], axis=1)
        ST = ST + (P * k[:, s])[..., None] * v[:, s][:, :, None, :]
    return y, ST


def abs_scale(r, w, k, v, state=None, kv_dtype: str = "f32"):
    """sigmoid(r_t) (S^abs_t |k_t|) with S^abs the recurrence on |k| |v|^T and |S_0|."""
    r, k, v = _f64(r, kv_dtype), _f64(k, kv_dtype), _f64(v, kv_dtype)
    w = np.asarray(w, np.float64)
    B, T, H, D = k.shape
    S = np.zeros((B, H, D, D)) if state is None else np.abs(np.array(state, np.float64))
    y = np.empty((B, T, H, D))
    ak, av = np.abs(k), np.abs(v)
    for t in range(T):
        S = w[:, t, :, :, None] * S + ak[:, t, :, :, None] * av[:, t, :, None, :]
        y[:, t] = _sigmoid(r[:, t]) * np.einsum("bhij,bhj->bhi", S, ak[:, t])
    return y, S
