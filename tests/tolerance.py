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
    rms = np.sqrt(np.mean(ref2 * ref2, axis=1, keepdims=True))
    a_row = 2.0 * ulp_bf16(rms) * 2.0 ** -8
    err = np.abs(gpu2 - ref2)
    u = ulp_bf16(ref2)
    tol_main = np.maximum(2.0 * u, 1e-2 * np.abs(ref2))
    tol = np.maximum(np.maximum(tol_main, a_row), 2.0 ** -126)
    finite = np.isfinite(ref2)
    bad = (~(err <= tol)) & finite
    bad |= (~np.isfinite(gpu2)) & finite
    floored = int(np.sum((err > tol_main) & (err <= tol)))
    max_ulp = float(np.max(np.where(finite, err / u, 0.0)))
    return {"ok": not bool(np.any(bad)), "n": int(ref2.size), "bad": int(np.sum(bad)),
            "max_ulp": max_ulp, "floored": floored,
            "first_bad": (np.argwhere(bad)[0].tolist() if np.any(bad) else None)}


def dw_fp32_check(gpu: np.ndarray, ref: np.ndarray) -> dict:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    tol = 1e-3 * np.maximum(np.abs(ref), rms)
    err = np.abs(gpu - ref)
    bad = ~(err <= tol)
    rel = float(np.max(err / np.maximum(np.maximum(np.abs(ref), rms), 1e-300))) if ref.size else 0
    return {"ok": not bool(np.any(bad)), "bad": int(np.sum(bad)), "max_rel": rel}


def rstd_check(gpu: np.ndarray, ref: np.ndarray) -> dict:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rel = np.abs(gpu - ref) / np.abs(ref)
    return {"ok": bool(np.all(rel <= 1e-5)), "max_rel": float(np.max(rel)) if rel.size else 0.0}
