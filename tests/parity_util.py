"""Shared helpers for the GPU parity tests: host<->device conversion and the
error metrics.

Metric for outputs. wkv_t is a convex combination of v, so a plain relative
error |out - ref| / |ref| is ill-conditioned where positive and negative values
cancel. The bar is instead  |out - ref| <= rtol * S_t  with
S_t = sum_i p_i |v_i| (the same weights applied to |v|, from the oracle run with
|v|), which is >= |ref| and equals it when all contributing v share a sign.
For bf16 outputs, the unavoidable rounding of the exact result to bf16 (up to
half a bf16 ulp, i.e. up to 2^-8 relative) is taken off first: the GPU value
must be within half an ulp of the float64 result plus rtol * S_t.

Metric for states (num, den, max_e): representation-free quantities are
compared -- log D = max_e + ln den to rtol absolute (a relative error of D),
num/den to rtol * (num/den scale) -- and max_e itself to rtol * max(1, |max_e|).
"""
from __future__ import annotations

import numpy as np
import torch

RTOL_F32 = 1e-5
RTOL_BF16 = 2e-3


def dev_f32(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()


def dev_bf16(codes):
    return torch.from_numpy(np.ascontiguousarray(codes, np.uint16).view(np.int16)).cuda().view(torch.bfloat16)


def host(t: torch.Tensor) -> np.ndarray:
    """A device tensor as float64 numpy (bf16 widened exactly)."""
    if t.dtype == torch.bfloat16:
        codes = t.view(torch.int16).cpu().numpy().view(np.uint16)
        return (codes.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return t.double().cpu().numpy()


def half_ulp_bf16(x):
    _, e = np.frexp(np.asarray(x, np.float64))
    return np.ldexp(1.0, e - 9)


def out_error(out, ref, scale, bf16_out=False):
    """Per-element error normalised by the scale (after bf16 rounding allowance)."""
    err = np.abs(np.asarray(out, np.float64) - ref)
    if bf16_out:
        err = np.maximum(err - half_ulp_bf16(ref), 0.0)
    return err / np.maximum(scale, 1e-300)


def assert_out(out, ref, scale, rtol, bf16_out=False, what="out"):
    assert out.shape == ref.shape, (out.shape, ref.shape)
    assert np.all(np.isfinite(out)), f"{what}: non-finite values"
    e = out_error(out, ref, scale, bf16_out)
    worst = float(e.max()) if e.size else 0.0
    if worst > rtol:
        idx = np.unravel_index(int(np.argmax(e)), e.shape)
        raise AssertionError(f"{what}: max normalised error {worst:.3e} > {rtol:.1e} at {idx}: "
                             f"gpu {out[idx]!r} ref {ref[idx]!r} scale {scale[idx]!r}")
    return worst


def assert_state(gs, rs, rs_abs_num, rtol, what="state"):
    gnum, gden, gmax = (np.asarray(x, np.float64) for x in gs)
    rnum, rden, rmax = (np.asarray(x, np.float64) for x in rs)
    assert np.all(np.isfinite(gnum)) and np.all(np.isfinite(gden)) and np.all(np.isfinite(gmax)), what
    assert np.all(gden > 0), f"{what}: den must be positive"
    logd = np.abs((gmax + np.log(gden)) - (rmax + np.log(rden)))
    assert logd.max() <= rtol, f"{what}: log D error {logd.max():.3e}"
    ratio_scale = np.maximum(np.asarray(rs_abs_num, np.float64) / rden, 1e-300)
    r = np.abs(gnum / gden - rnum / rden) / ratio_scale
    assert r.max() <= rtol, f"{what}: num/den error {r.max():.3e}"
    m = np.abs(gmax - rmax) / np.maximum(1.0, np.abs(rmax))
    assert m.max() <= rtol, f"{what}: max_e error {m.max():.3e}"
    return float(logd.max()), float(r.max()), float(m.max())
