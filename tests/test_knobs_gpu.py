"""Every tuning knob keeps the results right (GPU).

The knobs change launch shapes, pipeline depth, where the dw second pass runs, and whether
inputs are prefetched; y, rstd, dx and dg must not change at all (they are per row), and
dw must stay within its tolerance of the oracle.
"""
from __future__ import annotations

import itertools

import pytest
import torch

from gpu_util import Case, dev_to_f64, sample_rows
from synthetic import WORKLOADS
from tolerance import bf16_check, dw_fp32_check, rstd_check

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_norm_b200 as gn

KNOB_SETS = [
    dict(tail_reduce=t, chain_prefetch=c, l2_prefetch=l)
    for t, c, l in itertools.product((1, 2), (1, 2), (1, 2))
] + [
    dict(disable_pdl=1),
    dict(ctas_per_sm=1, stage_bytes=8192, max_stages=2),
    dict(ctas_per_sm=2, stage_bytes=98304),
    dict(fwd_direct=1),
    dict(fwd_direct=2),
    dict(bwd_direct=1),
    dict(bwd_direct=2),
    dict(fuse_fwd_bwd=1, bwd_direct=2),
    dict(fuse_fwd_bwd=2, bwd_direct=2),
]


@pytest.mark.parametrize("M,N", [(4099, 128), (700, 4096), (2500, 256), (1337, 40), (777, 16)])
@pytest.mark.parametrize("det", [True, False])
def test_knobs_do_not_change_results(M, N, det):
    case = Case(M, N, seed=23)
    ref = gn.gnorm_ckpt_step(case.x, case.g, case.w, case.eps, case.dy, dw_fp32=True,
                             deterministic=det)
    torch.cuda.synchronize()
    dw_oracle = case.oracle_dw()
    try:
        for knobs in KNOB_SETS:
            gn.gnorm_set_tuning(**knobs)
            out = gn.gnorm_ckpt_step(case.x, case.g, case.w, case.eps, case.dy, dw_fp32=True,
                                     deterministic=det)
            dx2, dg2, dw2 = gn.gnorm_bwd(case.dy, case.x, case.g, case.w, out[1], dw_fp32=True,
                                         deterministic=det)
            torch.cuda.synchronize()
            for a, b, name in zip(ref[:4], out[:4], ("y", "rstd", "dx", "dg")):
                assert torch.equal(a, b), (knobs, name)
            assert torch.equal(dx2, ref[2]) and torch.equal(dg2, ref[3]), knobs
            for dw in (out[4], dw2):
                rep = dw_fp32_check(dev_to_f64(dw), dw_oracle)
                assert rep["ok"], (knobs, rep)
    finally:
        gn.gnorm_set_tuning()
    assert gn.gnorm_device_error(reset=True) == 0


@pytest.mark.parametrize("M,N", [(1, 8), (37, 16), (1000, 40), (4099, 128), (2500, 256),
                                 (70001, 128)])
@pytest.mark.parametrize("w_fp32", [False, True])
@pytest.mark.parametrize("strided", [False, True])
def test_direct_and_staged_kernels_agree(M, N, w_fp32, strided):
    """The kernels that load rows straight into registers and the ones that stage them in
    shared memory do the same arithmetic in the same order: bitwise equal y, rstd, dx and dg,
    for packed and strided rows (x and g as the column halves of one buffer) and both weight
    types; dw (summed in another order) within its tolerance."""
    case = Case(M, N, seed=29)
    if strided:
        xg = torch.cat([case.x, case.g], dim=1)
        x, g = xg[:, :N], xg[:, N:]
    else:
        x, g = case.x, case.g
    w = case.w.float() if w_fp32 else case.w
    outs = []
    try:
        for mode in (1, 2):
            gn.gnorm_set_tuning(fwd_direct=mode)
            assert gn.gnorm_plan_query(0, M, N, True, 148)["direct_loads"] == (mode == 1)
            outs.append(gn.gnorm_fwd(x, g, w, case.eps))
        torch.cuda.synchronize()
    finally:
        gn.gnorm_set_tuning()
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    # the backward likewise: dx and dg bitwise equal, dw within its tolerance of the oracle
    dy = case.dy
    if strided:
        dyz = torch.cat([case.dy, torch.zeros_like(case.dy)], dim=1)
        dy = dyz[:, :N]
    rstd = outs[0][1]
    bwd = []
    try:
        for mode in (1, 2):
            gn.gnorm_set_tuning(bwd_direct=mode)
            assert gn.gnorm_plan_query(1, M, N, True, 148)["direct_loads"] == (mode == 1)
            bwd.append(gn.gnorm_bwd(dy, x, g, w, rstd, dw_fp32=True, deterministic=True))
        torch.cuda.synchronize()
    finally:
        gn.gnorm_set_tuning()
    assert torch.equal(bwd[0][0], bwd[1][0]) and torch.equal(bwd[0][1], bwd[1][1])
    dw_ref = case.oracle_dw()
    for out in bwd:
        rep = dw_fp32_check(dev_to_f64(out[2]), dw_ref)
        assert rep["ok"], rep
    assert gn.gnorm_device_error(reset=True) == 0


@pytest.mark.parametrize("det", [True, False])
def test_l2_prefetch_reaches_its_copies(det):
    """The L2 prefetch (flashinfer PR #8701, commit message: thread 0 warms L2 with the CTA's
    next row block) only issues copies when a CTA holds more row blocks than its ring: at
    368640 x 128 the staged forward has 2 stages of ~96 rows for ~13 blocks per CTA and the
    backward 3 stages for ~9, so most blocks prefetch the one a ring further on.  Results must
    not change at all (a prefetch writes no register and no memory) and must match the
    oracle on sampled rows and in dw."""
    wl = WORKLOADS["long_368640x128"]
    case = Case(wl.M, wl.N, seed=wl.seed, g_std=wl.g_std)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    outs = []
    try:
        for mode in (2, 1):
            gn.gnorm_set_tuning(l2_prefetch=mode)
            pf, pb = gn.gnorm_plan_query(0, wl.M, wl.N, det, sms), gn.gnorm_plan_query(1, wl.M, wl.N, det, sms)
            assert pf["l2_prefetch"] == (mode == 1) and pb["l2_prefetch"] == (mode == 1)
            assert not pf["direct_loads"] and not pb["direct_loads"]
            # more blocks per CTA than ring stages: the prefetch branch is taken
            assert pf["num_blocks"] > pf["grid"] * pf["stages"]
            assert pb["num_blocks"] > pb["grid"] * pb["stages"]
            y, rstd = gn.gnorm_fwd(case.x, case.g, case.w, case.eps)
            dx, dg, dw = gn.gnorm_bwd(case.dy, case.x, case.g, case.w, rstd, dw_fp32=True,
                                      deterministic=det)
            outs.append((y, rstd, dx, dg, dw))
        torch.cuda.synchronize()
    finally:
        gn.gnorm_set_tuning()
    for a, b, name in zip(outs[0][:4], outs[1][:4], ("y", "rstd", "dx", "dg")):
        assert torch.equal(a, b), name
    if det:
        assert torch.equal(outs[0][4], outs[1][4])
    y, rstd, dx, dg, dw = outs[1]
    rows = sample_rows(wl.M, n_random=4096)
    ry, rr, rdx, rdg = case.oracle_rows(rows)
    idx = torch.from_numpy(rows).cuda()
    for got, ref, name, chk in ((y, ry, "y", bf16_check), (rstd, rr, "rstd", rstd_check),
                                (dx, rdx, "dx", bf16_check), (dg, rdg, "dg", bf16_check)):
        rep = chk(dev_to_f64(got[idx]), ref)
        assert rep["ok"], (name, rep)
    rep = dw_fp32_check(dev_to_f64(dw), case.oracle_dw())
    assert rep["ok"], rep
    assert gn.gnorm_device_error(reset=True) == 0
