"""torch.autograd integration: the gated norm as a differentiable op.

``gated_rmsnorm(x, g, w, eps)`` runs gnorm_fwd and saves x, g, w and the FP32 rstd; its
backward runs gnorm_bwd.  The weight gradient comes back in w's dtype (BF16 or FP32; the
kernels accumulate it in FP32 either way).  Marshalling only: every step runs in the
library's CUDA kernels.
"""
from __future__ import annotations

import torch

from .gnorm import gnorm_bwd, gnorm_fwd

__all__ = ["GatedRMSNormFunction", "gated_rmsnorm", "GatedRMSNorm"]


class GatedRMSNormFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, g, w, eps: float, deterministic: bool):
        y, rstd = gnorm_fwd(x, g, w, eps)
        ctx.save_for_backward(x, g, w, rstd)
        ctx.deterministic = deterministic
        return y

    @staticmethod
    def backward(ctx, dy):
        x, g, w, rstd = ctx.saved_tensors
        dy = dy.contiguous() if not dy.is_contiguous() else dy
        dx, dg, dw = gnorm_bwd(dy, x, g, w, rstd, dw_fp32=w.dtype == torch.float32,
                               deterministic=ctx.deterministic)
        return dx, dg, dw, None, None


def gated_rmsnorm(x, g, w, eps: float = 1e-6, deterministic: bool = True):
    """y = x * rsqrt(mean(x^2) + eps) * w * g * sigmoid(g), differentiable in x, g and w."""
    return GatedRMSNormFunction.apply(x, g, w, eps, deterministic)


class GatedRMSNorm(torch.nn.Module):
    """Module form: a learnable weight of size N (BF16 by default, or FP32)."""

    def __init__(self, n: int, eps: float = 1e-6, *, dtype=torch.bfloat16, device=None,
                 deterministic: bool = True):
        super().__init__()
        self.weight = torch.nn.Parameter(torch.ones(n, dtype=dtype, device=device))
        self.eps = eps
        self.deterministic = deterministic

    def forward(self, x, g):
        return gated_rmsnorm(x, g, self.weight, self.eps, self.deterministic)
