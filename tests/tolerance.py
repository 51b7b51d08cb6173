"""Comparison rules for the CUDA path against the FP64 oracle.

BF16 outputs (y, dx, dg, BF16 dw): an element passes if
    |gpu - ref| <= max(2 * ulp_bf16(ref), 1e-2 * |ref|, a_row)
where ulp_bf16(v) = 2^(floor(log2|v|) - 7) and a_row = 2 * ulp_bf16(rms of the reference
row) * 2^-8 is a floor for results near zero (cancellation in dx, sigmoid(g) ~ 0 in y
and dg).  This is the stated bar "<= 2 BF16 ulp or rel 1e-2" plus that floor.  A second,
absolute floor of 2^-126 (the smallest normal FP32 and BF16 value) admits results that
the FP32 arithmetic flushes to zero: for g < -87, sigmoid(g) < 2^-126 is itself below
the normal range, so y and dg there are subnormal or zero.

FP32 dw: |dw_j - ref_j| <= 1e-3 * max(|ref_j|, rms(ref)).

Non-finite values (every rule): where the oracle is NaN the GPU must be NaN, and where the
oracle is +Inf or -Inf the GPU must be the same infinity; where the oracle is finite the
GPU must be finite.  Row and vector RMS floors are taken over the finite reference
entries only, so one NaN does not loosen or void the check of the rest of its row.

FP32 rstd: |gpu - ref| <= 1e-5 * ref.  Derivation: the kernel sums N squares in FP32 (a
sequential run of at most 32 per thread, then a tree), relative error below
(32 + log2(N)) * 2^-24 < 3e-6; rsqrtf adds 2 ulp (1.2e-7) and the square root halves
the relative error of its argument, so the total stays below 2e-6; 1e-5 leaves margin.
"""
from __future__ import annotations

import numpy as np


def ulp_bf16(v: np.ndarray) -> np.ndarray:
    a = np.abs(np.asarray(v, dtype=np.float64))
    tiny = 2.0 ** -126
    e = np.floor(np.log2(np.maximum(a, tiny)))
    return np.exp2(e - 7.0)


def nonfinite_mismatch(gpu: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """True where the oracle is NaN and the GPU is not, where the oracle is an infinity and
    the GPU is not that same infinity, or where the oracle is finite and the GPU is not."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    bad = np.isnan(ref) & ~np.isnan(gpu)
    bad |= np.isinf(ref) & ~(gpu == ref)
    bad |= np.isfinite(ref) & ~np.isfinite(gpu)
    return bad


def _rms_finite(ref: np.ndarray, axis=None, keepdims=False) -> np.ndarray:
    fin = np.isfinite(ref)
    r = np.where(fin, ref, 0.0)
    cnt = np.maximum(np.sum(fin, axis=axis, keepdims=keepdims), 1)
    return np.sqrt(np.sum(r * r, axis=axis, keepdims=keepdims) / cnt)


def bf16_check(gpu: np.ndarray, ref: np.ndarray, *, rows_axis: bool = True) -> dict:
    """Apply the BF16 rule; returns a report dict with 'ok'."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.ndim == 1 or not rows_axis:
        ref2 = ref.reshape(1, -1)
        gpu2 = gpu.reshape(1, -1)
    else:
        ref2, gpu2 = ref, gpu
    if ref2.size == 0:
        return {"ok": True, "n": 0, "bad": 0, "max_ulp": 0.0, "floored": 0}
    finite = np.isfinite(ref2)
    rms = _rms_finite(ref2, axis=1, keepdims=True)
    a_row = 2.0 * ulp_bf16(rms) * 2.0 ** -8
    with np.errstate(invalid="ignore"):
        err = np.where(finite, np.abs(gpu2 - ref2), 0.0)
    refz = np.where(finite, ref2, 1.0)
    u = ulp_bf16(refz)
    tol_main = np.maximum(2.0 * u, 1e-2 * np.abs(refz))
    tol = np.maximum(np.maximum(tol_main, a_row), 2.0 ** -126)
    bad = (~(err <= tol)) & finite
    bad |= nonfinite_mismatch(gpu2, ref2)
    floored = int(np.sum((err > tol_main) & (err <= tol) & finite))
    max_ulp = float(np.max(np.where(finite & np.isfinite(err), err / u, 0.0)))
    return {"ok": not bool(np.any(bad)), "n": int(ref2.size), "bad": int(np.sum(bad)),
            "max_ulp": max_ulp, "floored": floored, "nonfinite": int(np.sum(~finite)),
            "first_bad": (np.argwhere(bad)[0].tolist() if np.any(bad) else None)}


def dw_fp32_check(gpu: np.ndarray, ref: np.ndarray) -> dict:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    finite = np.isfinite(ref)
    rms = float(_rms_finite(ref)) if ref.size else 0.0
    refz = np.where(finite, ref, 0.0)
    tol = 1e-3 * np.maximum(np.abs(refz), rms)
    with np.errstate(invalid="ignore"):
        err = np.where(finite, np.abs(gpu - ref), 0.0)
    bad = (~(err <= tol)) & finite
    bad |= nonfinite_mismatch(gpu, ref)
    with np.errstate(invalid="ignore"):
        rel_all = np.where(finite, err / np.maximum(np.maximum(np.abs(refz), rms), 1e-300), 0.0)
    rel = float(np.max(rel_all)) if ref.size else 0.0
    return {"ok": not bool(np.any(bad)), "bad": int(np.sum(bad)), "max_rel": rel,
            "nonfinite": int(np.sum(~finite))}


def rstd_check(gpu: np.ndarray, ref: np.ndarray) -> dict:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    finite = np.isfinite(ref)
    with np.errstate(invalid="ignore", divide="ignore"):
        err = np.where(finite, np.abs(gpu - ref), 0.0)
        rel = np.where(finite & (ref != 0), err / np.abs(np.where(ref != 0, ref, 1.0)), 0.0)
    # a zero reference (an infinite row, r = 1/sqrt(inf)) must be matched exactly
    bad = (~(err <= 1e-5 * np.abs(np.where(finite, ref, 0.0)))) & finite
    bad |= nonfinite_mismatch(gpu, ref)
    return {"ok": not bool(np.any(bad)),
            "max_rel": float(np.max(np.where(np.isfinite(rel), rel, np.inf))) if rel.size else 0.0}
