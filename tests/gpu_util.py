"""Helpers shared by the GPU tests: device copies of the seeded inputs and oracle runs.

The inputs come from ``synthetic`` (BF16 bits); the expected values come only from the
FP64 oracle in ``oracle/``; the values under test come from the CUDA path through the
``gated_norm_b200`` binding of the C ABI.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from synthetic import bf16_bits_to_f64, make_inputs


def bits_to_dev(bits: np.ndarray, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16))
    return t.to(device).view(torch.bfloat16)


def dev_to_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def dev_to_f64(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return bf16_bits_to_f64(dev_to_bits(t))
    return t.detach().cpu().numpy().astype(np.float64)


class Case:
    """Seeded inputs on host (BF16 bits) and device (BF16 tensors)."""

    def __init__(self, M, N, *, seed=0, g_std=1.0, outlier_frac=0.0, eps=1e-6, device="cuda"):
        self.M, self.N, self.eps = M, N, eps
        self.host = make_inputs(M, N, seed=seed, g_std=g_std, outlier_frac=outlier_frac)
        self.x = bits_to_dev(self.host["x"], device)
        self.g = bits_to_dev(self.host["g"], device)
        self.dy = bits_to_dev(self.host["dy"], device)
        self.w = bits_to_dev(self.host["w"], device)

    def rows_f64(self, name, rows=None):
        b = self.host[name]
        return bf16_bits_to_f64(b if rows is None else b[rows])

    def oracle_rows(self, rows=None, rstd=None):
        """Oracle y, rstd, dx, dg on the given rows (all rows if None)."""
        x, g, dy = (self.rows_f64(k, rows) for k in ("x", "g", "dy"))
        w = bf16_bits_to_f64(self.host["w"])
        y, r = oracle.fwd(x, g, w, self.eps)
        dx, dg, _ = oracle.bwd(dy, x, g, w, r if rstd is None else rstd)
        return y, r, dx, dg

    def oracle_dw(self, chunk_rows=None):
        """Oracle dw over all rows, summed chunk by chunk (dw is a sum over rows)."""
        w = bf16_bits_to_f64(self.host["w"])
        if chunk_rows is None:
            chunk_rows = max(1, (1 << 22) // max(self.N, 1))
        dw = np.zeros(self.N)
        for r0 in range(0, self.M, chunk_rows):
            sl = slice(r0, min(self.M, r0 + chunk_rows))
            x, g, dy = (self.rows_f64(k, sl) for k in ("x", "g", "dy"))
            _, r = oracle.fwd(x, g, w, self.eps)
            dw += oracle.dw_rows(dy, x, g, r)
        return dw


def sample_rows(M: int, n_random: int = 2048, extra=(), seed: int = 1234) -> np.ndarray:
    """First and last 64 rows, `extra` rows and `n_random` seeded random rows (sorted)."""
    rng = np.random.default_rng(seed)
    parts = [np.arange(min(64, M)), np.arange(max(0, M - 64), M),
             np.asarray(extra, dtype=np.int64), rng.integers(0, M, min(n_random, M))]
    return np.unique(np.concatenate(parts).astype(np.int64))
