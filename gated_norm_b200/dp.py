"""Data-parallel plumbing for the weight gradient (torch.distributed over NCCL).

Rows of a data-parallel batch are independent, so the forward and the per-row backward
(dx, dg) need no communication.  dw is a sum over all rows of all ranks: each rank sums
its own rows (gnorm_bwd with an FP32 dw), then the ranks combine.  ``allreduce_dw`` does
that combine deterministically: it gathers the per-rank FP32 dw in rank order with
``all_gather_into_tensor`` and sums the rows with ``gnorm_dw_reduce`` (the library's
fixed-order kernel), so every rank ends with bitwise the same dw from run to run, whatever
reduction order the collective library would have used.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from .gnorm import gnorm_dw_reduce

__all__ = ["gather_dw", "allreduce_dw"]


def gather_dw(dw_local: torch.Tensor, group=None) -> torch.Tensor:
    """All ranks' FP32 dw stacked in rank order: a [world_size, N] tensor on every rank."""
    if dw_local.dtype != torch.float32 or dw_local.dim() != 1:
        raise ValueError("dw_local must be a 1-D FP32 tensor")
    world = dist.get_world_size(group)
    n = dw_local.numel()
    flat = torch.empty(world * n, dtype=torch.float32, device=dw_local.device)
    dist.all_gather_into_tensor(flat, dw_local.contiguous(), group=group)
    return flat.view(world, n)


def allreduce_dw(dw_local: torch.Tensor, *, dw_fp32: bool = True, out=None, group=None,
                 stream=None) -> torch.Tensor:
    """Deterministic cross-rank sum of the FP32 weight gradient (see module docstring)."""
    parts = gather_dw(dw_local, group)
    return gnorm_dw_reduce(parts, dw=out, dw_fp32=dw_fp32, stream=stream)
