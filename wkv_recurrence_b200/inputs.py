"""Seeded synthetic inputs for the WKV operator.

This module is shared by the CUDA-path tests, the benchmark and the oracle-side
tests. It holds no WKV arithmetic: only random draws, bf16 rounding of the
draws, and the workload shapes. Every array is produced on the host with
numpy, so the GPU side and the oracle side consume identical bytes.

Each tensor row (one batch entry / one decode stream / one decode step) is drawn
from its own generator, seeded by ``(seed, workload code, tensor code, row)``,
so any subset of rows can be regenerated without drawing the rest.

Workloads (names follow the operator's notation: keys ``k``, values ``v``,
per-channel decay ``w`` and bonus ``u``, the layout is ``[B, T, C]`` with the
channel axis fastest):

``tiny``      B=1, T=8, C=4 fp32, zero initial state (brute-force case)
``small``     B=1, T=64, C=768 fp32, zero initial state
``layer``     B=8, T=1024, C=768 fp32 (the MicroRWKV layer shape: 8 heads x 96)
``decode``    4096 streams x C=768 fp32; a 512-token prefix builds the state,
              then 256 one-token steps with fresh k, v
``long``      B=1, T=65536, C=2048 fp32; 1% of keys replaced by +-U(20, 60);
              w log-uniform in [1e-4, 4]
``mixed``     B=16, T=4096, C=4096; k and v rounded to bf16 (k = 2 * Student-t
              with 3 degrees of freedom, v ~ N(0, 1)); a nonzero random initial
              state; bf16 output

Distribution notation: ``N(mu, sigma)`` is mean and standard deviation.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# tensor codes for the per-row generators
_W, _U, _K, _V, _SNUM, _SDEN, _SMAX, _DK, _DV, _WT, _R = range(11)


@dataclass(frozen=True)
class Workload:
    name: str
    code: int
    B: int
    T: int
    C: int
    kv_dtype: str = "f32"          # "f32" or "bf16"
    out_dtype: str = "f32"
    state: str = "zero"            # "zero" or "random"
    k_dist: str = "normal"         # "normal", "spiky", "t3x2"
    w_dist: str = "lognormal"      # "lognormal" or "loguniform"
    decode_steps: int = 0          # one-token steps after the T-token prefix
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    "tiny": Workload("tiny", 10, B=1, T=8, C=4),
    "small": Workload("small", 11, B=1, T=64, C=768),
    "layer": Workload("layer", 12, B=8, T=1024, C=768),
    "decode": Workload("decode", 13, B=4096, T=512, C=768, decode_steps=256),
    "long": Workload("long", 14, B=1, T=65536, C=2048, k_dist="spiky",
                     w_dist="loguniform"),
    "mixed": Workload("mixed", 15, B=16, T=4096, C=4096, kv_dtype="bf16",
                      out_dtype="bf16", state="random", k_dist="t3x2"),
}


def _rng(seed: int, code: int, tensor: int, row: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(code), int(tensor), int(row)])


def _rng5(seed: int, code: int, tensor: int, row: int, blk: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(code), int(tensor), int(row), int(blk)])


# ---------------------------------------------------------------------------
# bf16 rounding of fp32 draws (round to nearest even), kept as raw 16-bit codes
# ---------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); return uint16 codes."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 codes to fp32 exactly."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------------------
# parameter and sequence draws
# ---------------------------------------------------------------------------

def draw_w(wl: Workload, seed: int = 0) -> np.ndarray:
    """Per-channel decay w, fp32 [C]."""
    g = _rng(seed, wl.code, _W, 0)
    if wl.w_dist == "loguniform":
        x = np.exp(g.uniform(np.log(1e-4), np.log(4.0), wl.C))
    else:
        x = np.clip(np.exp(g.normal(-1.0, 1.0, wl.C)), 1e-3, 8.0)
    return x.astype(np.float32)


def draw_u(wl: Workload, seed: int = 0) -> np.ndarray:
    """Per-channel bonus u ~ N(0, 0.5), fp32 [C]."""
    g = _rng(seed, wl.code, _U, 0)
    return g.normal(0.0, 0.5, wl.C).astype(np.float32)


_BLOCK_T = 512          # tokens per independently seeded block of a row


def _keys_block(wl: Workload, g: np.random.Generator, out: np.ndarray) -> None:
    n = out.size
    if wl.k_dist == "t3x2":
        # Student-t, 3 degrees of freedom, by its definition Z / sqrt(X/3) with
        # X a chi-square of 3 degrees (a sum of three squared standard normals)
        z = g.standard_normal((4, n), dtype=np.float32)
        x = z[1] * z[1] + z[2] * z[2] + z[3] * z[3]
        out.reshape(-1)[:] = np.float32(2.0) * z[0] / np.sqrt(x / np.float32(3.0))
        return
    g.standard_normal(dtype=np.float32, out=out.reshape(-1))
    if wl.k_dist == "spiky":
        flat = out.reshape(-1)
        hit = np.flatnonzero(g.random(n, dtype=np.float32) < np.float32(0.01))
        sign = np.where(g.random(hit.size) < 0.5, -1.0, 1.0)
        flat[hit] = (sign * g.uniform(20.0, 60.0, hit.size)).astype(np.float32)


def _pool_map(fn, items):
    items = list(items)
    if len(items) <= 1:
        for it in items:
            fn(it)
        return
    from concurrent.futures import ThreadPoolExecutor
    import os
    with ThreadPoolExecutor(max(1, min(16, os.cpu_count() or 1))) as ex:
        list(ex.map(fn, items))


def draw_kv_rows(wl: Workload, rows, seed: int = 0, T: int | None = None):
    """k, v for the given batch rows: arrays [len(rows), T, C].

    fp32 workloads give float32 arrays; bf16 workloads give uint16 bf16 codes.
    Each row is drawn in blocks of 512 tokens, each block from its own
    generator seeded by (seed, workload, tensor, row, block).
    """
    T = wl.T if T is None else T
    rows = list(rows)
    bf16 = wl.kv_dtype == "bf16"
    dt = np.uint16 if bf16 else np.float32
    k = np.empty((len(rows), T, wl.C), dt)
    v = np.empty((len(rows), T, wl.C), dt)
    nblk = max(1, -(-T // _BLOCK_T))

    def one(job):
        i, b, j = job
        t0, t1 = j * _BLOCK_T, min(T, (j + 1) * _BLOCK_T)
        kb = np.empty((t1 - t0, wl.C), np.float32)
        vb = np.empty((t1 - t0, wl.C), np.float32)
        _keys_block(wl, _rng5(seed, wl.code, _K, b, j), kb)
        _rng5(seed, wl.code, _V, b, j).standard_normal(dtype=np.float32, out=vb.reshape(-1))
        if bf16:
            kb, vb = f32_to_bf16_bits(kb), f32_to_bf16_bits(vb)
        k[i, t0:t1] = kb
        v[i, t0:t1] = vb

    _pool_map(one, [(i, b, j) for i, b in enumerate(rows) for j in range(nblk)])
    return k, v


def draw_kv(wl: Workload, seed: int = 0):
    return draw_kv_rows(wl, range(wl.B), seed)


def draw_wt_rows(wl: Workload, rows, seed: int = 0, T: int | None = None) -> np.ndarray:
    """Per-token decays w_t for the given rows, fp32 [len(rows), T, C], drawn
    per token from the workload's w distribution (log-normal exp(N(-1, 1))
    clipped to [1e-3, 8], or log-uniform in [1e-4, 4]); in 512-token blocks
    seeded by (seed, workload, tensor, row, block), like k and v."""
    T = wl.T if T is None else T
    rows = list(rows)
    out = np.empty((len(rows), T, wl.C), np.float32)
    nblk = max(1, -(-T // _BLOCK_T))

    def one(job):
        i, b, j = job
        t0, t1 = j * _BLOCK_T, min(T, (j + 1) * _BLOCK_T)
        g = _rng5(seed, wl.code, _WT, b, j)
        if wl.w_dist == "loguniform":
            x = np.exp(g.uniform(np.log(1e-4), np.log(4.0), (t1 - t0, wl.C)))
        else:
            x = np.clip(np.exp(g.normal(-1.0, 1.0, (t1 - t0, wl.C))), 1e-3, 8.0)
        out[i, t0:t1] = x.astype(np.float32)

    _pool_map(one, [(i, b, j) for i, b in enumerate(rows) for j in range(nblk)])
    return out


def draw_r_rows(wl: Workload, rows, seed: int = 0, T: int | None = None) -> np.ndarray:
    """Receptance r ~ N(0, 1) for the given rows, [len(rows), T, C] in the
    element type of k and v (uint16 bf16 codes for bf16 workloads)."""
    T = wl.T if T is None else T
    rows = list(rows)
    bf16 = wl.kv_dtype == "bf16"
    out = np.empty((len(rows), T, wl.C), np.uint16 if bf16 else np.float32)
    nblk = max(1, -(-T // _BLOCK_T))

    def one(job):
        i, b, j = job
        t0, t1 = j * _BLOCK_T, min(T, (j + 1) * _BLOCK_T)
        x = _rng5(seed, wl.code, _R, b, j).standard_normal((t1 - t0, wl.C), dtype=np.float32)
        out[i, t0:t1] = f32_to_bf16_bits(x) if bf16 else x

    _pool_map(one, [(i, b, j) for i, b in enumerate(rows) for j in range(nblk)])
    return out


def draw_state(wl: Workload, rows=None, seed: int = 0):
    """Initial state (num, den, max_e), each fp32 [len(rows), C], or None.

    "random" gives a nonzero state: den ~ U(1, 16), num = den * N(0, 0.5),
    max_e ~ N(2, 2). Any such triple is a valid state (den >= 1).
    """
    if wl.state != "random":
        return None
    rows = range(wl.B) if rows is None else list(rows)
    num = np.empty((len(rows), wl.C), np.float32)
    den = np.empty((len(rows), wl.C), np.float32)
    mx = np.empty((len(rows), wl.C), np.float32)
    for i, b in enumerate(rows):
        den[i] = _rng(seed, wl.code, _SDEN, b).uniform(1.0, 16.0, wl.C)
        num[i] = den[i] * _rng(seed, wl.code, _SNUM, b).normal(0.0, 0.5, wl.C)
        mx[i] = _rng(seed, wl.code, _SMAX, b).normal(2.0, 2.0, wl.C)
    return num, den, mx


_DEC_BLOCK = 256         # streams per independently seeded block of a decode token


def draw_decode_token(wl: Workload, step: int, rows=None, seed: int = 0):
    """Fresh k, v ~ N(0, 1) for one decode step: fp32 [len(rows), C].

    The streams are drawn in blocks of 256, each block from its own generator
    seeded by (seed, workload, tensor, step, block), so any subset of streams
    can be regenerated by drawing only the blocks that hold them.
    """
    rows = np.asarray(range(wl.B) if rows is None else list(rows), np.int64)
    k = np.empty((rows.size, wl.C), np.float32)
    v = np.empty((rows.size, wl.C), np.float32)

    def one(blk):
        n = min(_DEC_BLOCK, wl.B - int(blk) * _DEC_BLOCK)
        sel = np.flatnonzero(rows // _DEC_BLOCK == blk)
        local = rows[sel] - int(blk) * _DEC_BLOCK
        kb = _rng5(seed, wl.code, _DK, step, int(blk)).standard_normal((n, wl.C), dtype=np.float32)
        vb = _rng5(seed, wl.code, _DV, step, int(blk)).standard_normal((n, wl.C), dtype=np.float32)
        k[sel] = kb[local]
        v[sel] = vb[local]

    _pool_map(one, np.unique(rows // _DEC_BLOCK).tolist())
    return k, v


def random_case(B: int, T: int, C: int, seed: int, *, k_scale: float = 1.0,
                k_spike: float = 0.0, w_range=(1e-3, 8.0), u_sigma: float = 0.5,
                state: bool = False):
    """A generic random case for tests: fp32 k, v [B,T,C], w, u [C], state or None.

    w is log-uniform in ``w_range``; with ``k_spike`` > 0, 2% of keys are set
    to +-k_spike.
    """
    g = np.random.default_rng([int(seed), 99, B, T, C])
    w = np.exp(g.uniform(np.log(w_range[0]), np.log(w_range[1]), C)).astype(np.float32)
    u = g.normal(0.0, u_sigma, C).astype(np.float32)
    k = (k_scale * g.standard_normal((B, T, C))).astype(np.float32)
    if k_spike:
        m = g.random((B, T, C)) < 0.02
        k[m] = (np.where(g.random(int(m.sum())) < 0.5, -1.0, 1.0) * k_spike).astype(np.float32)
    v = g.standard_normal((B, T, C)).astype(np.float32)
    st = None
    if state:
        den = g.uniform(1.0, 16.0, (B, C)).astype(np.float32)
        num = (den * g.normal(0.0, 0.5, (B, C))).astype(np.float32)
        mx = g.normal(1.0, 2.0, (B, C)).astype(np.float32)
        st = (num, den, mx)
    return k, v, w, u, st


# ---------------------------------------------------------------------------
# the RWKV-v6 matrix-valued state ("RWKV-v6 Architecture", section
# "3. Matrix-Valued Hidden State")
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class V6Workload:
    name: str
    code: int
    B: int
    T: int
    H: int
    D: int
    kv_dtype: str = "f32"
    out_dtype: str = "f32"


V6_WORKLOADS = {
    # the MicroRWKV layer width (768 = 12 heads x 64) at its block length
    "v6": V6Workload("v6", 20, B=8, T=1024, H=12, D=64),
    "v6_bf16": V6Workload("v6_bf16", 21, B=8, T=1024, H=12, D=64, kv_dtype="bf16", out_dtype="bf16"),
}


def draw_v6(wl: V6Workload, seed: int = 0, T: int | None = None):
    """r, w, k, v [B, T, H, D]: r, k, v ~ N(0, 1) (bf16 codes for bf16
    workloads), w = exp(-exp(N(-1, 1))) fp32 (the page's decay form applied to
    a standard-normal projection shifted by -1). Each (tensor, batch row) from
    its own generator."""
    T = wl.T if T is None else T
    shape = (T, wl.H, wl.D)
    bf16 = wl.kv_dtype == "bf16"
    out = {}
    for name, code in (("r", 0), ("w", 1), ("k", 2), ("v", 3)):
        dt = np.float32 if (name == "w" or not bf16) else np.uint16
        arr = np.empty((wl.B,) + shape, dt)
        for b in range(wl.B):
            g = _rng(seed, wl.code, 100 + code, b)
            if name == "w":
                arr[b] = np.exp(-np.exp(g.normal(-1.0, 1.0, shape))).astype(np.float32)
            else:
                x = g.standard_normal(shape, dtype=np.float32)
                arr[b] = f32_to_bf16_bits(x) if bf16 else x
        out[name] = arr
    return out["r"], out["w"], out["k"], out["v"]
