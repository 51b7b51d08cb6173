"""Strided rows and an FP32 weight (GPU).

x and g as the two column halves of one [M, 2N] buffer (the gate packed with x), dx and dg
into the two halves of one gradient buffer, dy and y with padded rows.  Results must equal
the packed path bit for bit (same arithmetic), match the oracle, and leave the padding
between rows untouched.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from gpu_util import Case, dev_to_f64
from synthetic import bf16_bits_to_f64
from tolerance import bf16_check, dw_fp32_check

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_norm_b200 as gn

PAD = -7.0  # marks padding columns that no kernel may write


def _strided_layout(case):
    M, N = case.M, case.N
    xg = torch.empty(M, 2 * N, dtype=torch.bfloat16, device="cuda")
    xg[:, :N] = case.x
    xg[:, N:] = case.g
    dy_buf = torch.full((M, N + 24), PAD, dtype=torch.bfloat16, device="cuda")
    dy_buf[:, :N] = case.dy
    y_buf = torch.full((M, N + 8), PAD, dtype=torch.bfloat16, device="cuda")
    grad = torch.full((M, 2 * N + 16), PAD, dtype=torch.bfloat16, device="cuda")
    return dict(x=xg[:, :N], g=xg[:, N:], dy=dy_buf[:, :N], y=y_buf[:, :N], y_buf=y_buf,
                dx=grad[:, :N], dg=grad[:, N:2 * N], grad=grad)


# With the default plans, narrow rows with few rows per SM take the direct-load kernels
# (strided rows are plain loads there); (50000, 128)'s backward stages its blocks through
# 2-D tensor maps and (65, 4096) through one copy per row.  The staged kernels' strided
# paths at the other sizes are compared with the direct ones in test_knobs_gpu.py.
@pytest.mark.parametrize("M,N", [(1, 128), (257, 128), (4099, 136), (33, 256), (65, 4096),
                                 (300000, 8), (50000, 128)])
@pytest.mark.parametrize("det", [True, False])
def test_strided_equals_packed_and_oracle(M, N, det):
    case = Case(M, N, seed=41)
    L = _strided_layout(case)
    ref = gn.gnorm_ckpt_step(case.x, case.g, case.w, case.eps, case.dy, dw_fp32=True,
                             deterministic=det)
    out = gn.gnorm_ckpt_step(L["x"], L["g"], case.w, case.eps, L["dy"], y=L["y"], dx=L["dx"],
                             dg=L["dg"], dw_fp32=True, deterministic=det)
    torch.cuda.synchronize()
    for a, b, name in zip(ref[:4], out[:4], ("y", "rstd", "dx", "dg")):
        assert torch.equal(a, b.contiguous()), name
    if det:
        assert torch.equal(ref[4], out[4])
    assert torch.all(L["y_buf"][:, N:] == PAD)
    assert torch.all(L["grad"][:, 2 * N:] == PAD)
    ry, rr, rdx, rdg = case.oracle_rows()
    assert bf16_check(dev_to_f64(out[0].contiguous()), ry)["ok"]
    assert bf16_check(dev_to_f64(out[2].contiguous()), rdx)["ok"]
    assert bf16_check(dev_to_f64(out[3].contiguous()), rdg)["ok"]
    assert dw_fp32_check(dev_to_f64(out[4]), case.oracle_dw())["ok"]


@pytest.mark.parametrize("M,N", [(300, 128), (40, 4096), (129, 256)])
def test_fp32_weight(M, N):
    """An FP32 weight whose values are not BF16-representable; the oracle uses them exactly."""
    case = Case(M, N, seed=43)
    rng = np.random.default_rng(44)
    w32 = (1.0 + 0.1 * rng.standard_normal(N)).astype(np.float32)
    w = torch.from_numpy(w32).cuda()
    y, rstd, dx, dg, dw = gn.gnorm_ckpt_step(case.x, case.g, w, case.eps, case.dy, dw_fp32=True)
    torch.cuda.synchronize()
    import oracle
    x, g, dy = (bf16_bits_to_f64(case.host[k]) for k in ("x", "g", "dy"))
    ry, rr = oracle.fwd(x, g, w32.astype(np.float64), case.eps)
    rdx, rdg, rdw = oracle.bwd(dy, x, g, w32.astype(np.float64), rr)
    assert bf16_check(dev_to_f64(y), ry)["ok"]
    assert bf16_check(dev_to_f64(dx), rdx)["ok"]
    assert bf16_check(dev_to_f64(dg), rdg)["ok"]
    assert dw_fp32_check(dev_to_f64(dw), rdw)["ok"]


def test_strided_views_rejected_when_misaligned():
    buf = torch.zeros(16, 140, dtype=torch.bfloat16, device="cuda")
    x = buf[:, :128]  # row stride 140: rows would not start 16-byte aligned
    w = torch.ones(128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gn.GnormError) as e:
        gn.gnorm_fwd(x, x, w)
    assert "ALIGN" in str(e.value)
