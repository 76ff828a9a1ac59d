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
``abs_scale_*``         the same oracles run with |v| (and |num_in|): the
                        per-output scale sum_i p_i |v_i| used by the parity
                        metric.

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

def recurrence_forward(k, v, w, u, state=None, kv_dtype: str = "f32", threads: int = 0):
    """Float64 recurrence over [B, T, C] inputs.

    k, v: float32 arrays, or uint16 bf16 codes when kv_dtype == "bf16".
    w, u: float32 [C]. state: (num, den, max_e) arrays [B, C] or None (empty).
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
    lib.wkv_oracle_forward(B, T, C, _p(k), _p(v), code, _p(w), _p(u),
                           _p(si[0]), _p(si[1]), _p(si[2]), _p(out),
                           _p(so[0]), _p(so[1]), _p(so[2]), int(threads))
    return out, tuple(so)


def recurrence_step(state, k, v, w, u):
    """One float64 decode token for S streams: k, v float32 [S, C]; state arrays [S, C].

    Returns (out float64 [S, C], new state float64 triple).
    """
    lib = _load()
    k = np.ascontiguousarray(k, np.float32)
    v = np.ascontiguousarray(v, np.float32)
    S, C = k.shape
    si = [np.ascontiguousarray(s, np.float64) for s in state]
    out = np.empty((S, C), np.float64)
    so = [np.empty((S, C), np.float64) for _ in range(3)]
    lib.wkv_oracle_step(S, C, _p(k), _p(v), _p(np.ascontiguousarray(w, np.float32)),
                        _p(np.ascontiguousarray(u, np.float32)),
                        _p(si[0]), _p(si[1]), _p(si[2]), _p(out), _p(so[0]), _p(so[1]), _p(so[2]))
    return out, tuple(so)


# ---------------------------------------------------------------------------
# the equation as a direct sum (float64 numpy)
# ---------------------------------------------------------------------------

def _widen(x, kv_dtype):
    if kv_dtype == "bf16":
        return (np.asarray(x, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return np.asarray(x, np.float64)


def _exponent_matrix(T, w, u, k):
    """x[t, i] = k_i - (t-1-i) w for i < t, u + k_t for i = t, -inf for i > t (0-based)."""
    t = np.arange(T)[:, None]
    i = np.arange(T)[None, :]
    x = k[None, :] - (t - 1 - i) * w
    x = np.where(i < t, x, -np.inf)
    x[np.arange(T), np.arange(T)] = u + k
    return x


def direct_forward(k, v, w, u, state=None, kv_dtype: str = "f32"):
    """The equation for wkv_t summed directly, float64, for every (b, t, c).

    Returns (out [B, T, C], (num, den, max_e) [B, C]). O(B C T^2): small cases.
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
            x = _exponent_matrix(T, w[c], u[c], kc)
            if state is not None:
                n0, d0, m0 = (float(s[b, c]) for s in state)
                xs = m0 - np.arange(T) * w[c]          # state term at token t (0-based)
            else:
                n0 = d0 = 0.0
                xs = np.full(T, -np.inf)
            top = np.maximum(x.max(axis=1), xs)
            e = np.exp(x - top[:, None])
            es = np.exp(xs - top)
            out[b, :, c] = (e @ vc + es * n0) / (e.sum(axis=1) + es * d0)
            # state after T tokens: every token decays by (T-1-i) w, the state by T w
            y = kc - (T - 1 - np.arange(T)) * w[c]
            ys = (m0 - T * w[c]) if state is not None else -np.inf
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


def direct_output(kc, vc, w: float, u: float, t: int, state=None, kv_dtype: str = "f32") -> float:
    """wkv at 0-based token t of one channel, by the direct sum over tokens 0..t.

    kc, vc: that channel's keys and values over (at least) tokens 0..t.
    state: (num0, den0, m0) scalars or None.
    """
    kc = _widen(kc[: t + 1], kv_dtype)
    vc = _widen(vc[: t + 1], kv_dtype)
    w, u = float(w), float(u)
    i = np.arange(t + 1)
    x = kc - (t - 1 - i) * w
    x[t] = u + kc[t]
    if state is not None:
        n0, d0, m0 = (float(s) for s in state)
        xs = m0 - t * w
    else:
        n0 = d0 = 0.0
        xs = -np.inf
    top = max(x.max(), xs)
    e = np.exp(x - top)
    es = np.exp(xs - top)
    return float((e @ vc + es * n0) / (e.sum() + es * d0))


def decimal_forward(k, v, w, u, digits: int = 50):
    """The equation for wkv_t in ``digits``-digit decimal arithmetic (zero state).

    k, v: float32 [B, T, C]; w, u: float32 [C]. Every fp32 input converts to
    Decimal exactly. Returns out as a nested list of Decimal [B][T][C].
    """
    getcontext().prec = digits
    k = np.asarray(k, np.float32)
    v = np.asarray(v, np.float32)
    B, T, C = k.shape
    res = [[[None] * C for _ in range(T)] for _ in range(B)]
    for b in range(B):
        for c in range(C):
            wd, ud = Decimal(float(w[c])), Decimal(float(u[c]))
            kd = [Decimal(float(k[b, i, c])) for i in range(T)]
            vd = [Decimal(float(v[b, i, c])) for i in range(T)]
            for t in range(T):
                num = Decimal(0)
                den = Decimal(0)
                for i in range(t):
                    e = (kd[i] - (t - 1 - i) * wd).exp()
                    num += e * vd[i]
                    den += e
                e = (ud + kd[t]).exp()
                num += e * vd[t]
                den += e
                res[b][t][c] = num / den
    return res


# ---------------------------------------------------------------------------
# the per-output scale sum_i p_i |v_i| for the parity metric
# ---------------------------------------------------------------------------

def _abs_v(v, kv_dtype):
    if kv_dtype == "bf16":
        return (np.asarray(v, np.uint16) & np.uint16(0x7FFF)).astype(np.uint16)
    return np.abs(np.asarray(v, np.float32))


def abs_scale_forward(k, v, w, u, state=None, kv_dtype: str = "f32", threads: int = 0):
    """sum_i p_i |v_i| for every output, and the matching |num| state scale."""
    st = None
    if state is not None:
        st = (np.abs(np.asarray(state[0], np.float64)), state[1], state[2])
    return recurrence_forward(k, _abs_v(v, kv_dtype), w, u, st, kv_dtype, threads)


def abs_scale_step(state_abs, k, v, w, u):
    return recurrence_step(state_abs, k, np.abs(np.asarray(v, np.float32)), w, u)
