"""Seeded synthetic inputs for the SiLU-gated RMSNorm training path.

This module is shared by the CPU oracle's tests, the CUDA parity tests and the
benchmark.  It holds none of the operation's arithmetic: it draws random
numbers, rounds them to BF16 and describes the workloads.  Every tensor is
returned as raw BF16 bit patterns (``uint16``) so that the GPU path and the
oracle consume exactly the same bytes.

Recipe (the same for every workload):

* ``rng = numpy.random.default_rng(seed)``; draws in the order x, g, dy, w,
  each in FP32 with ``standard_normal``;
* ``g`` is multiplied by ``g_std`` (a standard deviation, not a variance);
* ``w = 1 + 0.1 * N(0, 1)`` over the N columns;
* if ``outlier_frac > 0``: ``round(outlier_frac * M)`` rows are picked with
  ``rng.permutation(M)`` (drawn after w) and their x is multiplied by
  ``outlier_scale`` in FP32;
* every tensor is then rounded to BF16 with round-to-nearest-even.

The row shapes mirror the workloads of flashinfer PR #8701
("perf(cake_rmsnorm_silu_gate_train): L2-prefetching extra-long forward on
SM107", Tables 1 and 2): rows are tokens x heads flattened, each row one
head-dim vector, BF16 inputs.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "f32_to_bf16_bits",
    "bf16_bits_to_f32",
    "bf16_bits_to_f64",
    "make_inputs",
    "make_workload_inputs",
    "make_cotangent",
]


def f32_to_bf16_bits(a) -> np.ndarray:
    """Round FP32 values to BF16 (round to nearest, ties to even); return bits.

    BF16 keeps the upper 16 bits of an IEEE binary32 word.  Rounding adds
    0x7FFF plus the lowest kept bit before truncating, which rounds halfway
    cases to the even neighbour.  NaN stays NaN (quiet bit forced); values
    that round past the largest finite BF16 become infinity, as IEEE requires.
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    keep_lsb = (u >> np.uint64(16)) & np.uint64(1)
    rounded = ((u + np.uint64(0x7FFF) + keep_lsb) >> np.uint64(16)).astype(np.uint16)
    is_nan = ((u & np.uint64(0x7F800000)) == np.uint64(0x7F800000)) & (
        (u & np.uint64(0x007FFFFF)) != np.uint64(0)
    )
    if np.any(is_nan):
        quiet = ((u >> np.uint64(16)) | np.uint64(0x0040)).astype(np.uint16)
        rounded = np.where(is_nan, quiet, rounded)
    return rounded


def bf16_bits_to_f32(bits) -> np.ndarray:
    """Widen BF16 bit patterns to FP32 exactly (shift into the high half)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Widen BF16 bit patterns to FP64 exactly."""
    return bf16_bits_to_f32(bits).astype(np.float64)


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: shape, input distributions and the ops it runs."""

    name: str
    M: int
    N: int
    g_std: float = 1.0
    outlier_frac: float = 0.0
    outlier_scale: float = 50.0
    eps: float = 1e-6
    seed: int = 0
    ops: tuple = field(default_factory=tuple)
    dw_fp32: tuple = (False,)
    deterministic: tuple = (True,)
    note: str = ""

    @property
    def rows(self) -> int:
        return self.M

    def scaled(self, M: int) -> "Workload":
        """The same distributions with a different row count."""
        return Workload(
            name=f"{self.name}[M={M}]", M=M, N=self.N, g_std=self.g_std,
            outlier_frac=self.outlier_frac, outlier_scale=self.outlier_scale,
            eps=self.eps, seed=self.seed, ops=self.ops, dw_fp32=self.dw_fp32,
            deterministic=self.deterministic, note=self.note,
        )


# The five workloads the implementation is measured and checked on.
WORKLOADS = {
    "small_1024x128": Workload(
        "small_1024x128", 1024, 128, ops=("fwd", "bwd"), dw_fp32=(False,),
        deterministic=(True,), note="small case; the oracle finishes in seconds",
    ),
    "linattn_65536x128": Workload(
        "linattn_65536x128", 65536, 128, ops=("fwd", "bwd", "ckpt"),
        dw_fp32=(False, True), deterministic=(True, False),
        note="per-head gated norm of a linear-attention output, 512 heads x 128 tokens",
    ),
    "long_368640x128": Workload(
        "long_368640x128", 368640, 128, g_std=2.0, ops=("fwd", "bwd"),
        dw_fp32=(True,), deterministic=(True, False),
        note="long row-count regime (about 1740 rows per SM on a 212-SM part)",
    ),
    "wide_16384x4096": Workload(
        "wide_16384x4096", 16384, 4096, outlier_frac=0.01, outlier_scale=50.0,
        ops=("fwd", "bwd", "ckpt"), dw_fp32=(False, True), deterministic=(True, False),
        note="wide rows; 1% of rows scaled by 50",
    ),
    "mid_262144x256": Workload(
        "mid_262144x256", 262144, 256, ops=("ckpt",), dw_fp32=(True,),
        deterministic=(True,), note="checkpointed step, bitwise repeatability over 10 runs",
    ),
}


def make_inputs(M: int, N: int, *, seed: int = 0, g_std: float = 1.0,
                outlier_frac: float = 0.0, outlier_scale: float = 50.0) -> dict:
    """Draw x, g, dy [M, N] and w [N] per the recipe; return BF16 bits.

    Also returns ``outlier_rows`` (sorted int64 row indices, possibly empty).
    """
    if M < 0 or N < 0:
        raise ValueError("M and N must be non-negative")
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, N), dtype=np.float32)
    g = rng.standard_normal((M, N), dtype=np.float32)
    if g_std != 1.0:
        g *= np.float32(g_std)
    dy = rng.standard_normal((M, N), dtype=np.float32)
    w = np.float32(1.0) + np.float32(0.1) * rng.standard_normal(N, dtype=np.float32)
    n_out = int(round(outlier_frac * M)) if outlier_frac > 0 else 0
    if n_out > 0:
        rows = np.sort(rng.permutation(M)[:n_out]).astype(np.int64)
        x[rows] *= np.float32(outlier_scale)
    else:
        rows = np.zeros(0, dtype=np.int64)
    return {
        "x": f32_to_bf16_bits(x),
        "g": f32_to_bf16_bits(g),
        "dy": f32_to_bf16_bits(dy),
        "w": f32_to_bf16_bits(w),
        "outlier_rows": rows,
    }


def make_workload_inputs(wl: Workload) -> dict:
    """``make_inputs`` with a workload's shape and distributions."""
    return make_inputs(wl.M, wl.N, seed=wl.seed, g_std=wl.g_std,
                       outlier_frac=wl.outlier_frac, outlier_scale=wl.outlier_scale)


def make_cotangent(M: int, N: int, *, seed: int) -> np.ndarray:
    """An independent BF16 upstream gradient (bits), for linearity checks."""
    rng = np.random.default_rng(seed)
    return f32_to_bf16_bits(rng.standard_normal((M, N), dtype=np.float32))
