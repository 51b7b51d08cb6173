"""gnorm_fwd_bwd: the forward and the backward of the same rows in one kernel (GPU).

The checkpointed step of flashinfer PR #8701 ("How the tables were measured": ckptg =
2 x forward + backward) ends with the recompute forward and the backward.  This library
runs those two as one kernel that reads x, g and dy once; its outputs must be bitwise those
of gnorm_fwd followed by gnorm_bwd (dw too in deterministic mode: the same plan sums the
same rows in the same order), for every row geometry, packed and strided rows, both
weight types, and they must match the FP64 oracle.
"""
from __future__ import annotations

import pytest
import torch

from gpu_util import Case, dev_to_f64
from tolerance import bf16_check, dw_fp32_check, rstd_check

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_norm_b200 as gn

# every staged geometry of the backward: N <= 32, <= 64, <= 128, <= 256, <= 512, <= 1024,
# <= 2048, <= 4096 (also 2056), <= 8192 (6144, 8192: xhat recomputed in pass 2), <= 16384
# (8200, 16384: u recomputed too); ragged row counts; 700 x 4096 has many blocks per CTA
SHAPES = [(300, 32), (1000, 64), (4099, 128), (2500, 256), (777, 136), (600, 512), (333, 1024),
          (97, 2048), (129, 2056), (700, 4096), (45, 6144), (23, 8192), (37, 8200), (19, 16384),
          (70001, 128), (16385, 256)]


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


def _same(a, b):
    return torch.equal(_bits(a), _bits(b))


@pytest.mark.parametrize("M,N", SHAPES)
@pytest.mark.parametrize("det", [True, False])
@pytest.mark.parametrize("dw_fp32", [True, False])
def test_fused_equals_forward_then_backward(M, N, det, dw_fp32):
    case = Case(M, N, seed=M + 3 * N)
    try:
        gn.gnorm_set_tuning(bwd_direct=2)  # the staged backward plan (the fused kernel)
        assert not gn.gnorm_plan_query(1, M, N, det, torch.cuda.get_device_properties(0)
                                       .multi_processor_count)["direct_loads"]
        y, rstd = gn.gnorm_fwd(case.x, case.g, case.w, case.eps)
        dx, dg, dw = gn.gnorm_bwd(case.dy, case.x, case.g, case.w, rstd, dw_fp32=dw_fp32,
                                  deterministic=det)
        fy, frstd, fdx, fdg, fdw = gn.gnorm_fwd_bwd(case.x, case.g, case.w, case.eps, case.dy,
                                                    dw_fp32=dw_fp32, deterministic=det)
        torch.cuda.synchronize()
    finally:
        gn.gnorm_set_tuning()
    for a, b, name in ((y, fy, "y"), (rstd, frstd, "rstd"), (dx, fdx, "dx"), (dg, fdg, "dg")):
        assert _same(a, b), name
    if det:
        assert _same(dw, fdw)
    ref = case.oracle_dw()
    rep = (dw_fp32_check if dw_fp32 else bf16_check)(dev_to_f64(fdw), ref)
    assert rep["ok"], rep
    assert gn.gnorm_device_error(reset=True) == 0


@pytest.mark.parametrize("M,N", [(1537, 136), (4099, 128), (40, 4096), (2500, 256)])
def test_fused_matches_oracle(M, N):
    case = Case(M, N, seed=11, g_std=2.0)
    try:
        gn.gnorm_set_tuning(bwd_direct=2)
        y, rstd, dx, dg, dw = gn.gnorm_fwd_bwd(case.x, case.g, case.w, case.eps, case.dy,
                                               dw_fp32=True)
        torch.cuda.synchronize()
    finally:
        gn.gnorm_set_tuning()
    ry, rr, rdx, rdg = case.oracle_rows()
    for got, ref, name, chk in ((y, ry, "y", bf16_check), (rstd, rr, "rstd", rstd_check),
                                (dx, rdx, "dx", bf16_check), (dg, rdg, "dg", bf16_check)):
        rep = chk(dev_to_f64(got), ref)
        assert rep["ok"], (name, rep)
    rep = dw_fp32_check(dev_to_f64(dw), case.oracle_dw())
    assert rep["ok"], rep


@pytest.mark.parametrize("w_fp32", [False, True])
def test_fused_strided_rows_and_fp32_weight(w_fp32):
    """x and g as the column halves of one [M, 2N] buffer, dx and dg as the halves of one
    gradient buffer, y written into a wider buffer: the same bits as the packed calls."""
    M, N = 3001, 256
    case = Case(M, N, seed=5)
    w = case.w.float() if w_fp32 else case.w
    xg = torch.cat([case.x, case.g], dim=1)
    x, g = xg[:, :N], xg[:, N:]
    grad = torch.zeros(M, 2 * N, dtype=torch.bfloat16, device="cuda")
    ybuf = torch.zeros(M, N + 64, dtype=torch.bfloat16, device="cuda")
    try:
        gn.gnorm_set_tuning(bwd_direct=2, fuse_fwd_bwd=2)  # packed, as separate kernels
        ref = gn.gnorm_ckpt_step(case.x, case.g, w, case.eps, case.dy, dw_fp32=True)
        gn.gnorm_set_tuning(bwd_direct=2, fuse_fwd_bwd=1)
        out = gn.gnorm_fwd_bwd(x, g, w, case.eps, case.dy, y=ybuf[:, :N], dx=grad[:, :N],
                               dg=grad[:, N:], dw_fp32=True)
        torch.cuda.synchronize()
    finally:
        gn.gnorm_set_tuning()
    for a, b, name in zip(ref[:4], (ybuf[:, :N], out[1], grad[:, :N], grad[:, N:]),
                          ("y", "rstd", "dx", "dg")):
        assert _same(a.contiguous(), b.contiguous()), name
    assert _same(ref[4], out[4])
    assert torch.all(ybuf[:, N:] == 0)  # the padding past each row is untouched


@pytest.mark.parametrize("M,N", [(65536, 128), (4099, 256), (700, 4096)])
@pytest.mark.parametrize("det", [True, False])
def test_ckpt_step_fused_and_unfused_agree(M, N, det):
    """The checkpointed step with its recompute forward fused into the backward and with
    three separate kernels: bitwise the same y, rstd, dx, dg (and dw when deterministic)."""
    case = Case(M, N, seed=M % 97 + N)
    outs = []
    try:
        for fuse in (1, 2):
            gn.gnorm_set_tuning(fuse_fwd_bwd=fuse, bwd_direct=2)
            outs.append(gn.gnorm_ckpt_step(case.x, case.g, case.w, case.eps, case.dy,
                                           dw_fp32=True, deterministic=det))
        torch.cuda.synchronize()
    finally:
        gn.gnorm_set_tuning()
    for a, b, name in zip(outs[0][:4], outs[1][:4], ("y", "rstd", "dx", "dg")):
        assert _same(a, b), name
    if det:
        assert _same(outs[0][4], outs[1][4])
    rep = dw_fp32_check(dev_to_f64(outs[0][4]), case.oracle_dw())
    assert rep["ok"], rep


def test_fused_with_direct_backward_plan_runs_two_kernels():
    """Few rows per SM: the backward loads rows into registers, so gnorm_fwd_bwd runs the
    forward and the backward as two kernels -- same results."""
    case = Case(1024, 128, seed=2)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert gn.gnorm_plan_query(1, 1024, 128, True, sms)["direct_loads"]
    y, rstd = gn.gnorm_fwd(case.x, case.g, case.w, case.eps)
    dx, dg, dw = gn.gnorm_bwd(case.dy, case.x, case.g, case.w, rstd, dw_fp32=True)
    out = gn.gnorm_fwd_bwd(case.x, case.g, case.w, case.eps, case.dy, dw_fp32=True)
    torch.cuda.synchronize()
    for a, b in zip((y, rstd, dx, dg, dw), out):
        assert _same(a, b)


def test_fused_argument_errors():
    from gated_norm_b200.gnorm import GnormError
    case = Case(64, 128, seed=1)
    with pytest.raises(GnormError):  # an output overlapping an input
        gn.gnorm_fwd_bwd(case.x, case.g, case.w, case.eps, case.dy, y=case.x)
    with pytest.raises(GnormError):
        gn.gnorm_fwd_bwd(case.x, case.g, case.w, float("nan"), case.dy)
    empty = torch.empty(0, 128, dtype=torch.bfloat16, device="cuda")
    dw = torch.full((128,), 7.0, device="cuda")
    gn.gnorm_fwd_bwd(empty, empty, case.w, case.eps, empty, dw=dw, dw_fp32=True)
    torch.cuda.synchronize()
    assert torch.all(dw == 0)  # M == 0: dw = 0
