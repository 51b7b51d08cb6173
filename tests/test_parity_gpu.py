"""CUDA path against the FP64 oracle, element by element (GPU).

Small and ragged shapes are compared in full; the five workloads are compared in full
where the oracle is quick (1024x128, 65536x128) and otherwise on sampled rows, with dw
always over all rows.  Tolerances are those of tests/tolerance.py.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from gpu_util import Case, dev_to_f64, sample_rows
from synthetic import WORKLOADS
from tolerance import bf16_check, dw_fp32_check, rstd_check

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_norm_b200 as gn

SMALL_SHAPES = [
    (1, 8), (3, 24), (7, 64), (2, 120), (257, 128), (1000, 136), (129, 256), (33, 520),
    (65, 1024), (17, 2056), (40, 4096), (5, 8200), (3, 16384), (300, 32), (1537, 128),
]


def _check_fwd(case, y, rstd, rows=None):
    ry, rr, _, _ = case.oracle_rows(rows)
    yg = dev_to_f64(y if rows is None else y[torch.from_numpy(rows).to(y.device)])
    rg = dev_to_f64(rstd if rows is None else rstd[torch.from_numpy(rows).to(rstd.device)])
    rep_y = bf16_check(yg, ry)
    rep_r = rstd_check(rg, rr)
    assert rep_y["ok"], f"y: {rep_y}"
    assert rep_r["ok"], f"rstd: {rep_r}"
    return rep_y


def _check_bwd(case, dx, dg, rows=None):
    _, _, rdx, rdg = case.oracle_rows(rows)
    sel = (lambda t: t) if rows is None else (lambda t: t[torch.from_numpy(rows).to(t.device)])
    rep_dx = bf16_check(dev_to_f64(sel(dx)), rdx)
    rep_dg = bf16_check(dev_to_f64(sel(dg)), rdg)
    assert rep_dx["ok"], f"dx: {rep_dx}"
    assert rep_dg["ok"], f"dg: {rep_dg}"


def _check_dw(case, dw, dw_fp32):
    ref = case.oracle_dw()
    got = dev_to_f64(dw)
    rep = dw_fp32_check(got, ref) if dw_fp32 else bf16_check(got, ref)
    assert rep["ok"], f"dw ({'fp32' if dw_fp32 else 'bf16'}): {rep}"


@pytest.mark.parametrize("M,N", SMALL_SHAPES)
def test_fwd_small(M, N):
    case = Case(M, N, seed=M * 7 + N)
    y, rstd = gn.gnorm_fwd(case.x, case.g, case.w, case.eps)
    torch.cuda.synchronize()
    _check_fwd(case, y, rstd)


@pytest.mark.parametrize("M,N", SMALL_SHAPES)
@pytest.mark.parametrize("dw_fp32", [False, True])
@pytest.mark.parametrize("det", [True, False])
def test_bwd_small(M, N, dw_fp32, det):
    case = Case(M, N, seed=M * 11 + N, g_std=2.0)
    y, rstd = gn.gnorm_fwd(case.x, case.g, case.w, case.eps)
    dx, dg, dw = gn.gnorm_bwd(case.dy, case.x, case.g, case.w, rstd, dw_fp32=dw_fp32,
                              deterministic=det)
    torch.cuda.synchronize()
    _check_bwd(case, dx, dg)
    _check_dw(case, dw, dw_fp32)


@pytest.mark.parametrize("M,N", [(257, 128), (40, 4096), (129, 256)])
def test_bwd_with_gpu_rstd(M, N):
    """The backward alone: the oracle consumes the GPU's FP32 rstd."""
    case = Case(M, N, seed=5)
    _, rstd = gn.gnorm_fwd(case.x, case.g, case.w, case.eps)
    dx, dg, _ = gn.gnorm_bwd(case.dy, case.x, case.g, case.w, rstd)
    torch.cuda.synchronize()
    _, _, rdx, rdg = case.oracle_rows(None, rstd=dev_to_f64(rstd))
    assert bf16_check(dev_to_f64(dx), rdx)["ok"]
    assert bf16_check(dev_to_f64(dg), rdg)["ok"]


@pytest.mark.parametrize("M,N", [(1, 8), (257, 128), (33, 520), (40, 4096)])
@pytest.mark.parametrize("det", [True, False])
def test_ckpt_small(M, N, det):
    case = Case(M, N, seed=3)
    y, rstd, dx, dg, dw = gn.gnorm_ckpt_step(case.x, case.g, case.w, case.eps, case.dy,
                                             dw_fp32=True, deterministic=det)
    torch.cuda.synchronize()
    _check_fwd(case, y, rstd)
    _check_bwd(case, dx, dg)
    _check_dw(case, dw, True)


def test_extreme_gate_and_zero_rows():
    """Large gates (|g| up to 80, where sigmoid(g) is still a normal FP32 number) and
    all-zero rows (r = 1/sqrt(eps)), compared element by element."""
    from gpu_util import dev_to_bits
    case = Case(64, 256, seed=9)
    g = torch.linspace(-80, 80, 64 * 256, device="cuda").reshape(64, 256).to(torch.bfloat16)
    x = case.x.clone()
    x[5].zero_()
    x[17].zero_()
    case.host["g"] = dev_to_bits(g)
    case.host["x"] = dev_to_bits(x)
    case.g, case.x = g, x
    y, rstd = gn.gnorm_fwd(case.x, case.g, case.w, case.eps)
    dx, dg, dw = gn.gnorm_bwd(case.dy, case.x, case.g, case.w, rstd, dw_fp32=True)
    torch.cuda.synchronize()
    _check_fwd(case, y, rstd)
    _check_bwd(case, dx, dg)
    _check_dw(case, dw, True)


def test_saturated_gate():
    """|g| >= 90: sigmoid(g) is 0 or 1 in FP32.  Outputs stay finite; for g <= -90 they are
    below 1e-30 in magnitude (the true values are under 1e-36); for g >= 90 y equals the
    gate limit rmsnorm(x) * w * g within the BF16 rule."""
    N = 128
    case = Case(8, N, seed=10)
    gv = torch.tensor([-200.0, -120.0, -100.0, -90.0, 90.0, 100.0, 120.0, 200.0], device="cuda")
    g = gv[:, None].expand(8, N).contiguous().to(torch.bfloat16)
    y, rstd = gn.gnorm_fwd(case.x, g, case.w, case.eps)
    dx, dg, dw = gn.gnorm_bwd(case.dy, case.x, g, case.w, rstd, dw_fp32=True)
    torch.cuda.synchronize()
    for t in (y, dx, dg, dw):
        assert torch.all(torch.isfinite(t.float()))
    assert float(y[:4].float().abs().max()) < 1e-30
    assert float(dg[:4].float().abs().max()) < 1e-30
    xhat = torch.nn.functional.rms_norm(case.x.double(), (N,), eps=case.eps)
    ref = (xhat * case.w.double() * g.double())[4:]
    from tolerance import bf16_check
    assert bf16_check(dev_to_f64(y[4:]), ref.cpu().numpy())["ok"]


def test_zero_rows_m0():
    N = 128
    x = torch.empty(0, N, dtype=torch.bfloat16, device="cuda")
    w = torch.ones(N, dtype=torch.bfloat16, device="cuda")
    y, rstd = gn.gnorm_fwd(x, x, w, 1e-6)
    assert y.shape == (0, N) and rstd.shape == (0,)
    for fp32 in (False, True):
        dw = torch.full((N,), 7.0, dtype=torch.float32 if fp32 else torch.bfloat16, device="cuda")
        gn.gnorm_bwd(x, x, x, w, rstd, dw=dw, dw_fp32=fp32)
        torch.cuda.synchronize()
        assert torch.all(dw == 0)


# ------------------------------------------------------------------ the five workloads

def _workload_case(name, M=None):
    wl = WORKLOADS[name]
    return Case(M or wl.M, wl.N, seed=wl.seed, g_std=wl.g_std, outlier_frac=wl.outlier_frac,
                eps=wl.eps), wl


@pytest.mark.parametrize("name", ["small_1024x128", "linattn_65536x128"])
def test_workload_full_compare(name):
    case, wl = _workload_case(name)
    for det in wl.deterministic:
        for fp32 in wl.dw_fp32:
            y, rstd, dx, dg, dw = gn.gnorm_ckpt_step(case.x, case.g, case.w, case.eps, case.dy,
                                                     dw_fp32=fp32, deterministic=det)
            torch.cuda.synchronize()
            _check_fwd(case, y, rstd)
            _check_bwd(case, dx, dg)
            _check_dw(case, dw, fp32)


@pytest.mark.parametrize("name", ["long_368640x128", "wide_16384x4096", "mid_262144x256"])
def test_workload_sampled(name):
    """Full-size launch as the benchmark runs it; sampled rows, dw over all rows."""
    case, wl = _workload_case(name)
    rows = sample_rows(case.M, extra=case.host["outlier_rows"])
    dw_ref = case.oracle_dw()
    for det in wl.deterministic:
        for fp32 in wl.dw_fp32:
            if "ckpt" in wl.ops:
                y, rstd, dx, dg, dw = gn.gnorm_ckpt_step(case.x, case.g, case.w, case.eps,
                                                         case.dy, dw_fp32=fp32,
                                                         deterministic=det)
            else:
                y, rstd = gn.gnorm_fwd(case.x, case.g, case.w, case.eps)
                dx, dg, dw = gn.gnorm_bwd(case.dy, case.x, case.g, case.w, rstd, dw_fp32=fp32,
                                          deterministic=det)
            torch.cuda.synchronize()
            _check_fwd(case, y, rstd, rows)
            _check_bwd(case, dx, dg, rows)
            got = dev_to_f64(dw)
            rep = dw_fp32_check(got, dw_ref) if fp32 else bf16_check(got, dw_ref)
            assert rep["ok"], f"dw: {rep}"


@pytest.mark.parametrize("name", ["long_368640x128", "wide_16384x4096", "mid_262144x256"])
def test_workload_sampled_fused(name):
    """The forward fused into the backward (gnorm_fwd_bwd, the checkpointed step's second
    half, which the benchmark times at every large workload) at full size: sampled rows,
    dw over all rows."""
    case, wl = _workload_case(name)
    rows = sample_rows(case.M, extra=case.host["outlier_rows"])
    dw_ref = case.oracle_dw()
    for det in wl.deterministic:
        y, rstd, dx, dg, dw = gn.gnorm_fwd_bwd(case.x, case.g, case.w, case.eps, case.dy,
                                               dw_fp32=True, deterministic=det)
        torch.cuda.synchronize()
        _check_fwd(case, y, rstd, rows)
        _check_bwd(case, dx, dg, rows)
        rep = dw_fp32_check(dev_to_f64(dw), dw_ref)
        assert rep["ok"], f"dw: {rep}"
    assert gn.gnorm_device_error(reset=True) == 0
