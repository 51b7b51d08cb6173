"""gnorm_dw_reduce: the fixed-order sum of FP32 partial rows (GPU).

This is the step that combines per-rank FP32 dw in data-parallel training; the expected
value is the FP64 sum of the same rows.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from tolerance import bf16_check, dw_fp32_check

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_norm_b200 as gn


@pytest.mark.parametrize("P,N", [(1, 8), (2, 128), (8, 4096), (148, 256), (1000, 136)])
@pytest.mark.parametrize("dw_fp32", [True, False])
def test_matches_fp64_sum(P, N, dw_fp32):
    rng = np.random.default_rng(P * 31 + N)
    parts = rng.standard_normal((P, N)).astype(np.float32)
    ref = parts.astype(np.float64).sum(axis=0)
    dev = torch.from_numpy(parts).cuda()
    dw = gn.gnorm_dw_reduce(dev, dw_fp32=dw_fp32)
    torch.cuda.synchronize()
    got = dw.double().cpu().numpy()
    rep = dw_fp32_check(got, ref) if dw_fp32 else bf16_check(got, ref)
    assert rep["ok"], rep
    again = gn.gnorm_dw_reduce(dev, dw_fp32=dw_fp32)
    torch.cuda.synchronize()
    assert torch.equal(dw.view(torch.uint8), again.view(torch.uint8))  # fixed order


def test_zero_partials_give_zero():
    dw = torch.full((64,), 3.0, device="cuda")
    gn.gnorm_dw_reduce(torch.empty(0, 64, device="cuda"), dw=dw)
    torch.cuda.synchronize()
    assert torch.all(dw == 0)


def test_single_rank_combine_is_identity():
    """With one rank the deterministic combine returns that rank's dw exactly."""
    dw_local = torch.randn(512, device="cuda")
    out = gn.gnorm_dw_reduce(dw_local.view(1, -1))
    torch.cuda.synchronize()
    assert torch.equal(out, dw_local)


def test_allreduce_dw_single_rank_process_group():
    """gated_norm_b200.dp.allreduce_dw end to end in a world-size-1 NCCL process group: the
    gather returns this rank's row and the fixed-order sum is bitwise gnorm_dw_reduce of it
    (and, for one FP32 row, the row itself)."""
    import socket

    import torch.distributed as dist

    from gated_norm_b200.dp import allreduce_dw
    from gpu_util import Case

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    case = Case(4099, 256, seed=3)
    _, rstd = gn.gnorm_fwd(case.x, case.g, case.w, case.eps)
    _, _, dw_local = gn.gnorm_bwd(case.dy, case.x, case.g, case.w, rstd, dw_fp32=True)
    torch.cuda.synchronize()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                            world_size=1, device_id=torch.device("cuda", 0))
    try:
        for fp32 in (True, False):
            got = allreduce_dw(dw_local, dw_fp32=fp32)
            ref = gn.gnorm_dw_reduce(dw_local.view(1, -1), dw_fp32=fp32)
            torch.cuda.synchronize()
            assert torch.equal(got.view(torch.uint8), ref.view(torch.uint8)), fp32
        assert torch.equal(allreduce_dw(dw_local), dw_local)
        dist.barrier()
    finally:
        dist.destroy_process_group()
