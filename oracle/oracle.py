"""CPU oracle for the RWKV WKV operator (float64).

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the product path. It shares no code
with the CUDA library (no common headers, tables or helpers); the only thing
both sides share is the seeded input module, which holds no WKV arithmetic.

Source of truth: "Linear attention without writing a CUDA kernel" (page 1),
section "The recurrence":

* the equation for wkv_t (a weighted mean of v: weight e^{-(t-1-i)w + k_i} for
  an earlier token i, e^{u + k_t} for the current token), and
* the carried (numerator, denominator, max_exponent) state that turns the sum
  into a constant-cost step.

Functions
---------
``direct_forward``      the equation written out as a sum, float64, with the
                        largest exponent subtracted before exponentiating
                        (a log-sum-exp shift, which leaves the ratio unchanged).
                        O(T^2) per channel: the definition.
``direct_output``       one output (b, t, c) by the same sum, O(t): for sampled
                        checks at full size.
``decimal_forward``     the same sum in 50-digit decimal arithmetic (tiny cases).
``recurrence_forward``  the carried-state recurrence in float64 C (OpenMP over
                        channels): the O(T) oracle used at full size. Pinned to
                        the sum by the tests.
``recurrence_step``     one decode token for S streams, same recurrence.
``recurrence_backward`` the gradients of sum(g * wkv) with respect to k, v,
                        w, u and the state passed in, by the chain rule run
                        backwards through the same recurrence (float64 C), with
                        the magnitude scale of each gradient.
``abs_scale_*``         the same oracles run with |v| (and |num_in|): the
                        per-output scale sum_i p_i |v_i| used by the parity
                        metric.

Two extensions, from "RWKV-v6 Architecture: Attention-Free Linear
Transformers" (all functions above take them as optional arguments):

* ``w_t`` ([B, T, C], section "2. Dynamic Data-Dependent Decay"): a per-token
  decay in place of the per-channel w. It sits where w sits in the step
  function: token t's advance multiplies the state by e^{-w_t}. So an earlier
  token i reaches the output of token t with exponent
  k_i - (w_{i+1} + ... + w_{t-1}), a state passed in with m0 - (w_1 + ... +
  w_{t-1}), and the state after T tokens holds token i with
  k_i - (w_{i+1} + ... + w_T) (1-based). With w_t = w for every token this is
  the equation above.
* ``r`` ([B, T, C], the receptance of the v6 page's readout and of the
  Time-Mixing block of "RWKV: Merging Transformer Training with RNN Speed"):
  the output is gated, y_t = sigmoid(r_t) * wkv_t. The state is not gated.

Readings where the page is silent (each also listed in the design notes):

* the empty state is (num, den, max_e) = (0, 0, -inf);
* a state passed in, (num0, den0, m0), stands for the pair N0 = num0 e^{m0},
  D0 = den0 e^{m0} carried in front of token 1, and is used at token 1 without
  decay, exactly like the recurrence uses its state before decaying it. In the
  sum it enters as one more term with exponent m0 - (t-1) w (1-based t);
* the state after T tokens is reported in the form the recurrence produces:
  max_e = the largest exponent contributing to it, num = N_T e^{-max_e},
  den = D_T e^{-max_e}.

Parity unpinned: none. Every function here is pinned by the not-gpu tests
(closed forms, special cases reducing to a library softmax, brute force in
decimal arithmetic, invariants); see tests/test_oracle_pins.py.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from decimal import Decimal, getcontext

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wkv_oracle.c")
_LIB = os.path.join(_HERE, "_build", "libwkv_oracle.so")
_lib = None

F32, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile the C recurrence (gcc, -O2, OpenMP, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        os.makedirs(os.path.dirname(_LIB), exist_ok=True)
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off",
                        "-fno-fast-math", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"],
                       check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        lib.wkv_oracle_forward.argtypes = [I64, I64, I64, P, P, I, P, P, P, P, P, P, P, P, P, I]
        lib.wkv_oracle_forward.restype = None
        lib.wkv_oracle_step.argtypes = [I64, I64, P, P, P, P, P, P, P, P, P, P, P]
        lib.wkv_oracle_step.restype = None
        lib.wkv_oracle_max_threads.restype = ctypes.c_int
        lib.wkv_oracle_forward_ext.argtypes = [I64, I64, I64, P, P, I, P, P, P, P, P, P, P, P, P, P, P, I]
        lib.wkv_oracle_forward_ext.restype = None
        lib.wkv_oracle_step_ext.argtypes = [I64, I64, P, P, P, I, P, P, P, P, P, P, P, P, P]
        lib.wkv_oracle_step_ext.restype = None
        lib.wkv_oracle_backward.argtypes = [I64, I64, I64, P, P, I] + [P] * 20 + [I]
        lib.wkv_oracle_backward.restype = None
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().wkv_oracle_max_threads())


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _kv_arrays(k, v, kv_dtype):
    if kv_dtype == "bf16":
        k = np.ascontiguousarray(k, np.uint16)
        v = np.ascontiguousarray(v, np.uint16)
        return k, v, BF16
    return np.ascontiguousarray(k, np.float32), np.ascontiguousarray(v, np.float32), F32


# ---------------------------------------------------------------------------
# the recurrence (float64 C)
# ---------------------------------------------------------------------------

def recurrence_forward(k, v, w, u, state=None, kv_dtype: str = "f32", threads: int = 0, w_t=None, r=None):
    """Float64 recurrence over [B, T, C] inputs.

    k, v: float32 arrays, or uint16 bf16 codes when kv_dtype == "bf16".
    w, u: float32 [C]. state: (num, den, max_e) arrays [B, C] or None (empty).
    w_t: None or float32 [B, T, C], the per-token decay that replaces w.
    r: None or [B, T, C] receptance (the element type of k and v): out = sigmoid(r) wkv.
    Returns (out float64 [B, T, C], (num, den, max_e) float64 [B, C]).
    """
    lib = _load()
    k, v, code = _kv_arrays(k, v, kv_dtype)
    B, T, C = k.shape
    w = np.ascontiguousarray(w, np.float32)
    u = np.ascontiguousarray(u, np.float32)
    out = np.empty((B, T, C), np.float64)
    so = [np.empty((B, C), np.float64) for _ in range(3)]
    si = [None, None, None]
    if state is not None:
        si = [np.ascontiguousarray(np.broadcast_to(s, (B, C)), np.float64) for s in state]
    if w_t is None and r is None:
        lib.wkv_oracle_forward(B, T, C, _p(k), _p(v), code, _p(w), _p(u),
                               _p(si[0]), _p(si[1]), _p(si[2]), _p(out),
                               _p(so[0]), _p(so[1]), _p(so[2]), int(threads))
        return out, tuple(so)
    wt = None if w_t is None else np.ascontiguousarray(np.broadcast_to(w_t, (B, T, C)), np.float32)
    rr = None
    if r is not None:
        rr = np.ascontiguousarray(r, np.uint16 if kv_dtype == "bf16" else np.float32)
        assert rr.shape == (B, T, C)
    lib.wkv_oracle_forward_ext(B, T, C, _p(k), _p(v), code, _p(w), _p(wt), _p(u), _p(rr),
                               _p(si[0]), _p(si[1]), _p(si[2]), _p(out),
                               _p(so[0]), _p(so[1]), _p(so[2]), int(threads))
    return out, tuple(so)


def recurrence_step(state, k, v, w, u, r=None):
    """One float64 decode token for S streams: k, v float32 [S, C]; state arrays [S, C].

    w: float32 [C], or [S, C] (this step's per-token decay of every stream).
    r: None or float32 [S, C] receptance (out = sigmoid(r) wkv).
    Returns (out float64 [S, C], new state float64 triple).
    """
    lib = _load()
    k = np.ascontiguousarray(k, np.float32)
    v = np.ascontiguousarray(v, np.float32)
    S, C = k.shape
    si = [np.ascontiguousarray(s, np.float64) for s in state]
    out = np.empty((S, C), np.float64)
    so = [np.empty((S, C), np.float64) for _ in range(3)]
    w = np.ascontiguousarray(w, np.float32)
    u = np.ascontiguousarray(u, np.float32)
    if w.ndim == 1 and r is None:
        lib.wkv_oracle_step(S, C, _p(k), _p(v), _p(w), _p(u),
                            _p(si[0]), _p(si[1]), _p(si[2]), _p(out), _p(so[0]), _p(so[1]), _p(so[2]))
        return out, tuple(so)
    per_stream = int(w.ndim == 2)
    if per_stream:
        assert w.shape == (S, C)
    rr = None if r is None else np.ascontiguousarray(r, np.float32)
    lib.wkv_oracle_step_ext(S, C, _p(k), _p(v), _p(w), per_stream, _p(u), _p(rr),
                            _p(si[0]), _p(si[1]), _p(si[2]), _p(out), _p(so[0]), _p(so[1]), _p(so[2]))
    return out, tuple(so)


def recurrence_backward(k, v, w, u, gout, state=None, kv_dtype: str = "f32", threads: int = 0):
    """Gradients of sum(gout * wkv) by the float64 backward recurrence.

    gout: [B, T, C] (float64 or float32), dL/d wkv. No loss term on the final
    state. Returns two dicts, the gradients and their scales (the same
    formulas on magnitudes: the sum of |terms| of each gradient):
      dk, dv [B, T, C]; dw, du [C] (summed over the batch rows);
      dnum, dden, dmax [B, C] (the state passed in; zeros without one).
    """
    lib = _load()
    k, v, code = _kv_arrays(k, v, kv_dtype)
    B, T, C = k.shape
    w = np.ascontiguousarray(w, np.float32)
    u = np.ascontiguousarray(u, np.float32)
    g = np.ascontiguousarray(gout, np.float64)
    assert g.shape == (B, T, C)
    si = [None, None, None]
    if state is not None:
        si = [np.ascontiguousarray(np.broadcast_to(s, (B, C)), np.float64) for s in state]
    d = {n: np.zeros(sh) for n, sh in (("dk", (B, T, C)), ("dv", (B, T, C)), ("dw", (C,)), ("du", (C,)),
                                        ("dnum", (B, C)), ("dden", (B, C)), ("dmax", (B, C)))}
    sc = {n: np.zeros_like(a) for n, a in d.items()}
    lib.wkv_oracle_backward(B, T, C, _p(k), _p(v), code, _p(w), _p(u), _p(si[0]), _p(si[1]), _p(si[2]), _p(g),
                            _p(d["dk"]), _p(d["dv"]), _p(d["dw"]), _p(d["du"]),
                            _p(d["dnum"]), _p(d["dden"]), _p(d["dmax"]),
                            _p(sc["dk"]), _p(sc["dv"]), _p(sc["dw"]), _p(sc["du"]),
                            _p(sc["dnum"]), _p(sc["dden"]), _p(sc["dmax"]), int(threads))
    return d, sc


# ---------------------------------------------------------------------------
# the equation as a direct sum (float64 numpy)
# ---------------------------------------------------------------------------

def _widen(x, kv_dtype):
    if kv_dtype == "bf16":
        return (np.asarray(x, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return np.asarray(x, np.float64)


def _decay_sums(T, w, w_t):
    """P[t] = w_1 + ... + w_t over 1-based tokens, as a 0-based array P[0..T-1]
    (P[t] = (t+1) w for a constant decay), float64."""
    if w_t is None:
        return (np.arange(T) + 1.0) * float(w)
    return np.cumsum(np.asarray(w_t, np.float64))


def _exponent_matrix(T, u, k, P):
    """x[t, i] = k_i - (P[t-1] - P[i]) for i < t (the decays of tokens i+1..t-1),
    u + k_t for i = t, -inf for i > t (0-based)."""
    t = np.arange(T)[:, None]
    i = np.arange(T)[None, :]
    Pprev = np.concatenate([[0.0], P[:-1]])          # P[t-1], with P[-1] = 0
    x = k[None, :] - (Pprev[:, None] - P[None, :])
    x = np.where(i < t, x, -np.inf)
    x[np.arange(T), np.arange(T)] = u + k
    return x


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-np.asarray(x, np.float64)))


def direct_forward(k, v, w, u, state=None, kv_dtype: str = "f32", w_t=None, r=None):
    """The equation for wkv_t summed directly, float64, for every (b, t, c).

    w_t: None or [B, T, C] per-token decay; r: None or [B, T, C] receptance
    (out = sigmoid(r) wkv). Returns (out [B, T, C], (num, den, max_e) [B, C]).
    O(B C T^2): small cases.
    """
    kf, vf = _widen(k, kv_dtype), _widen(v, kv_dtype)
    B, T, C = kf.shape
    w = np.asarray(w, np.float64)
    u = np.asarray(u, np.float64)
    out = np.empty((B, T, C))
    num_o = np.empty((B, C))
    den_o = np.empty((B, C))
    max_o = np.empty((B, C))
    for b in range(B):
        for c in range(C):
            kc, vc = kf[b, :, c], vf[b, :, c]
            P = _decay_sums(T, w[c], None if w_t is None else np.asarray(w_t)[b, :, c])
            Pprev = np.concatenate([[0.0], P[:-1]])
            x = _exponent_matrix(T, u[c], kc, P)
            if state is not None:
                n0, d0, m0 = (float(s[b, c]) for s in state)
                xs = m0 - Pprev                         # state term at token t (0-based)
            else:
                n0 = d0 = 0.0
                xs = np.full(T, -np.inf)
            top = np.maximum(x.max(axis=1), xs) if T else xs
            e = np.exp(x - top[:, None])
            es = np.exp(xs - top)
            out[b, :, c] = (e @ vc + es * n0) / (e.sum(axis=1) + es * d0)
            if r is not None:
                out[b, :, c] *= _sigmoid(_widen(np.asarray(r)[b, :, c], kv_dtype))
            # state after T tokens: token i decayed by tokens i+1..T, the state by all T
            PT = P[-1] if T else 0.0
            y = kc - (PT - P)
            ys = (m0 - PT) if state is not None else -np.inf
            mx = max(y.max() if T else -np.inf, ys)
            if mx == -np.inf:
                num_o[b, c], den_o[b, c], max_o[b, c] = 0.0, 0.0, -np.inf
                continue
            ey = np.exp(y - mx)
            eys = np.exp(ys - mx)
            num_o[b, c] = ey @ vc + eys * n0
            den_o[b, c] = ey.sum() + eys * d0
            max_o[b, c] = mx
    return out, (num_o, den_o, max_o)


def direct_output(kc, vc, w: float, u: float, t: int, state=None, kv_dtype: str = "f32", w_t=None, r=None) -> float:
    """wkv at 0-based token t of one channel, by the direct sum over tokens 0..t.

    kc, vc: that channel's keys and values over (at least) tokens 0..t.
    state: (num0, den0, m0) scalars or None. w_t: None or that channel's
    per-token decays (at least tokens 0..t); r: None or its receptance at t.
    """
    kc = _widen(kc[: t + 1], kv_dtype)
    vc = _widen(vc[: t + 1], kv_dtype)
    u = float(u)
    P = _decay_sums(t + 1, w, None if w_t is None else np.asarray(w_t)[: t + 1])
    Pprev_t = P[t - 1] if t > 0 else 0.0
    x = kc - (Pprev_t - P)
    x[t] = u + kc[t]
    if state is not None:
        n0, d0, m0 = (float(s) for s in state)
        xs = m0 - Pprev_t
    else:
        n0 = d0 = 0.0
        xs = -np.inf
    top = max(x.max(), xs)
    e = np.exp(x - top)
    es = np.exp(xs - top)
    y = float((e @ vc + es * n0) / (e.sum() + es * d0))
    if r is not None:
        y *= float(_sigmoid(_widen(np.asarray([r]), kv_dtype)[0]))
    return y


def decimal_forward(k, v, w, u, digits: int = 50, w_t=None, r=None):
    """The equation for wkv_t in ``digits``-digit decimal arithmetic (zero state).

    k, v: float32 [B, T, C]; w, u: float32 [C]; w_t: None or float32 [B, T, C];
    r: None or float32 [B, T, C] (out = wkv / (1 + e^{-r})). Every fp32 input
    converts to Decimal exactly. Returns out as a nested list of Decimal [B][T][C].
    """
    getcontext().prec = digits
    k = np.asarray(k, np.float32)
    v = np.asarray(v, np.float32)
    B, T, C = k.shape
    res = [[[None] * C for _ in range(T)] for _ in range(B)]
    for b in range(B):
        for c in range(C):
            ud = Decimal(float(u[c]))
            if w_t is None:
                wd = [Decimal(float(w[c]))] * T
            else:
                wd = [Decimal(float(np.float32(w_t[b, i, c]))) for i in range(T)]
            kd = [Decimal(float(k[b, i, c])) for i in range(T)]
            vd = [Decimal(float(v[b, i, c])) for i in range(T)]
            for t in range(T):
                num = Decimal(0)
                den = Decimal(0)
                for i in range(t):
                    decay = sum(wd[i + 1:t], Decimal(0))       # tokens i+1 .. t-1
                    e = (kd[i] - decay).exp()
                    num += e * vd[i]
                    den += e
                e = (ud + kd[t]).exp()
                num += e * vd[t]
                den += e
                y = num / den
                if r is not None:
                    y = y / (Decimal(1) + (-Decimal(float(np.float32(r[b, t, c])))).exp())
                res[b][t][c] = y
    return res


# ---------------------------------------------------------------------------
# the per-output scale sum_i p_i |v_i| for the parity metric
# ---------------------------------------------------------------------------

def _abs_v(v, kv_dtype):
    if kv_dtype == "bf16":
        return (np.asarray(v, np.uint16) & np.uint16(0x7FFF)).astype(np.uint16)
    return np.abs(np.asarray(v, np.float32))


def abs_scale_forward(k, v, w, u, state=None, kv_dtype: str = "f32", threads: int = 0, w_t=None, r=None):
    """sum_i p_i |v_i| for every output (times sigmoid(r) when gated), and the
    matching |num| state scale."""
    st = None
    if state is not None:
        st = (np.abs(np.asarray(state[0], np.float64)), state[1], state[2])
    return recurrence_forward(k, _abs_v(v, kv_dtype), w, u, st, kv_dtype, threads, w_t=w_t, r=r)


def abs_scale_step(state_abs, k, v, w, u, r=None):
    return recurrence_step(state_abs, k, np.abs(np.asarray(v, np.float32)), w, u, r=r)
