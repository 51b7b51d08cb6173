"""FP64 CPU oracle for the SiLU-gated RMSNorm training forward and backward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or links
this module.  It is used by ``tests/``, by ``__graft_entry__.smoke()`` and by the
CPU baseline leg of ``bench.py``.  It shares no code with the CUDA kernels and
never imports the ``gated_norm_b200`` package.

What it computes
----------------
The subject page, flashinfer PR #8701 ("perf(cake_rmsnorm_silu_gate_train):
L2-prefetching extra-long forward on SM107", PR description), names the
operation "Cake's SiLU-gated RMSNorm training kernel".  Its section "How the
tables were measured" names kernels with the same semantics (FLA
``rms_norm_gated``, mamba_ssm ``rmsnorm_fn``), which normalise a row first and
then gate it.  The page prints no formula; this oracle takes the plain reading:

    forward, per row m of x[M, N] with gate g[M, N] and weight w[N]:
        r_m   = 1 / sqrt( (1/N) * sum_j x_mj^2 + eps )      (rstd, saved)
        y_mj  = x_mj * r_m * w_j * g_mj * sigmoid(g_mj)

    backward, with upstream gradient dy[M, N], using the saved r_m:
        xhat  = x * r,   s = g * sigmoid(g)  (= silu(g)),   u = dy * w * s
        c_m   = (1/N) * sum_j u_mj * xhat_mj
        dx    = r * (u - xhat * c)
        dg    = dy * xhat * w * sigmoid(g) * (1 + g * (1 - sigmoid(g)))
        dw_j  = sum_m dy_mj * xhat_mj * s_mj

dx is the derivative of sum(dy * y) with respect to x through r (the chain
rule on r = (mean(x^2) + eps)^-1/2); dg is dy * xhat * w times the derivative
of silu; dw sums the same product over rows.  The checkpointed step ("ckptg" /
"stepg_f32" in the page's list of operations) is two forward calls followed
by one backward call.

Inputs are the exact BF16 values widened to FP64; every result is FP64.  The
arithmetic follows the definitions above in their stated order with whole-array
numpy operations (``numpy.sum`` / ``numpy.mean`` as the only reductions); there
is no blocking or fusion.  Where the pages leave a step open, the reading taken
is stated next to the function.
"""
from __future__ import annotations

import numpy as np

__all__ = ["sigmoid", "silu", "fwd", "bwd", "dw_rows", "ckpt_step"]


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def sigmoid(t) -> np.ndarray:
    """Logistic function 1 / (1 + e^-t), in FP64.

    For t < 0 the equal form e^t / (1 + e^t) is used so that e^-t never
    overflows; NaN propagates.
    """
    t = _f64(t)
    out = np.empty_like(t)
    pos = t >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-t[pos]))
    neg = ~pos
    e = np.exp(t[neg])
    out[neg] = e / (1.0 + e)
    return out


def silu(t) -> np.ndarray:
    """SiLU (swish) gate t * sigmoid(t)."""
    t = _f64(t)
    return t * sigmoid(t)


def fwd(x, g, w, eps: float):
    """Forward: returns (y[M, N], rstd[M]) in FP64.

    Readings: one normalisation group is the whole row; eps sits inside the
    square root; there is no bias; the weight multiplies the normalised row
    before the gate.
    """
    x, g, w = _f64(x), _f64(g), _f64(w)
    ms = np.mean(x * x, axis=1)
    rstd = 1.0 / np.sqrt(ms + eps)
    y = x * rstd[:, None] * w[None, :] * g * sigmoid(g)
    return y, rstd


def bwd(dy, x, g, w, rstd):
    """Backward: returns (dx[M, N], dg[M, N], dw[N]) in FP64.

    ``rstd`` is the forward's saved reciprocal RMS per row (either the
    oracle's own or one produced elsewhere), used as given.
    """
    dy, x, g, w, rstd = _f64(dy), _f64(x), _f64(g), _f64(w), _f64(rstd)
    r = rstd[:, None]
    xhat = x * r
    sig = sigmoid(g)
    s = g * sig
    u = dy * w[None, :] * s
    c = np.mean(u * xhat, axis=1)
    dx = r * (u - xhat * c[:, None])
    dg = dy * xhat * w[None, :] * sig * (1.0 + g * (1.0 - sig))
    dw = np.sum(dy * xhat * s, axis=0)
    return dx, dg, dw


def dw_rows(dy, x, g, rstd):
    """The weight gradient over the given rows only: sum_m dy * xhat * silu(g).

    dw is a sum over rows, so the dw of a large input is the sum of this
    function over any split of its rows; tests use that to bound memory.
    """
    dy, x, g, rstd = _f64(dy), _f64(x), _f64(g), _f64(rstd)
    xhat = x * rstd[:, None]
    return np.sum(dy * xhat * (g * sigmoid(g)), axis=0)


def ckpt_step(x, g, w, eps: float, dy):
    """Checkpointed step: forward, forward again (recompute), backward.

    The second forward recomputes the same values as the first, so the
    outputs are (y, rstd) of the second call and (dx, dg, dw) of the backward
    that consumes that call's rstd.
    """
    y, rstd = fwd(x, g, w, eps)
    y, rstd = fwd(x, g, w, eps)
    dx, dg, dw = bwd(dy, x, g, w, rstd)
    return y, rstd, dx, dg, dw
