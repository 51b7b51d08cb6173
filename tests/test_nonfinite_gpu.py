"""Non-finite and saturating inputs through the CUDA path, against the oracle (GPU).

The operation is "Cake's SiLU-gated RMSNorm training kernel" (flashinfer PR #8701, PR
description) with the semantics of the comparator kernels named in its section "How the
tables were measured" (FLA rms_norm_gated, mamba_ssm rmsnorm_fn), which propagate NaN.
Reading taken: NaN and infinities follow IEEE arithmetic through the definition, in the
oracle and on the GPU alike; the sigmoid saturates to 0 or 1 for large finite |g| without
producing NaN.  Each case plants NaN, an infinity or a huge finite value at chosen places
(distinct rows and columns, so that what stays finite is still checked element by
element) and compares every output with the FP64 oracle: NaN where the oracle has NaN,
the same infinity where it has one, and the usual tolerances elsewhere.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from gpu_util import Case, bits_to_dev, dev_to_f64
from synthetic import f32_to_bf16_bits
from tolerance import bf16_check, dw_fp32_check, rstd_check

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_norm_b200 as gn

NAN, PINF, NINF = 0x7FC0, 0x7F80, 0xFF80


def _bits(v: float) -> int:
    return int(f32_to_bf16_bits(np.array([v], dtype=np.float32))[0])


# name -> list of (tensor, row or None for w, column, BF16 bits)
PLANTS = {
    "x_nan": [("x", 3, 5, NAN)],
    "x_inf": [("x", 7, 9, PINF)],
    "g_nan": [("g", 11, 2, NAN)],
    "g_pinf": [("g", 13, 17, PINF)],
    "g_ninf": [("g", 19, 23, NINF)],
    "g_saturated": [("g", 2, 1, _bits(1e30)), ("g", 4, 3, _bits(-1e30)),
                    ("g", 6, 6, _bits(100.0)), ("g", 8, 8, _bits(-100.0)),
                    ("g", 10, 12, _bits(3.0e7))],
    "dy_nan": [("dy", 29, 31, NAN)],
    "w_nan": [("w", None, 37, NAN)],
    "mixed": [("g", 11, 2, NAN), ("dy", 29, 31, NAN), ("g", 13, 17, PINF),
              ("g", 19, 23, NINF), ("g", 2, 1, _bits(1e30)), ("g", 4, 3, _bits(-1e30))],
}

# (M, N, knobs): the direct-load kernels, the staged kernels on the same narrow rows, and
# the staged kernels on wide rows.
KERNELS = {
    "direct_257x128": (257, 128, {}),
    "staged_257x128": (257, 128, {"fwd_direct": 2, "bwd_direct": 2}),
    "staged_40x4096": (40, 4096, {}),
}


def _as_int(t):
    """Bits of a BF16 or FP32 tensor (NaN compares equal to itself as bits)."""
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


def _planted_case(M, N, plant):
    case = Case(M, N, seed=101)
    for name, row, col, bits in PLANTS[plant]:
        arr = case.host[name]
        if row is None:
            arr[col] = bits
        else:
            arr[row, col] = bits
    for name in ("x", "g", "dy", "w"):
        setattr(case, name, bits_to_dev(case.host[name]))
    return case


@pytest.mark.parametrize("plant", sorted(PLANTS))
@pytest.mark.parametrize("kernels", sorted(KERNELS))
@pytest.mark.parametrize("det", [True, False])
@pytest.mark.parametrize("dw_fp32", [True, False])
def test_nonfinite_inputs_match_oracle(plant, kernels, det, dw_fp32):
    M, N, knobs = KERNELS[kernels]
    case = _planted_case(M, N, plant)
    try:
        gn.gnorm_set_tuning(**knobs)
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        direct = kernels.startswith("direct")
        assert gn.gnorm_plan_query(0, M, N, det, sms)["direct_loads"] == direct
        assert gn.gnorm_plan_query(1, M, N, det, sms)["direct_loads"] == direct
        y, rstd = gn.gnorm_fwd(case.x, case.g, case.w, case.eps)
        dx, dg, dw = gn.gnorm_bwd(case.dy, case.x, case.g, case.w, rstd, dw_fp32=dw_fp32,
                                  deterministic=det)
        ck = gn.gnorm_ckpt_step(case.x, case.g, case.w, case.eps, case.dy, dw_fp32=dw_fp32,
                                deterministic=det)
        torch.cuda.synchronize()
    finally:
        gn.gnorm_set_tuning()
    ry, rr, rdx, rdg = case.oracle_rows()
    rdw = case.oracle_dw()
    with np.errstate(invalid="ignore", over="ignore"):
        reports = {
            "y": bf16_check(dev_to_f64(y), ry),
            "rstd": rstd_check(dev_to_f64(rstd), rr),
            "dx": bf16_check(dev_to_f64(dx), rdx),
            "dg": bf16_check(dev_to_f64(dg), rdg),
            "dw": (dw_fp32_check if dw_fp32 else bf16_check)(dev_to_f64(dw), rdw),
        }
    bad = {k: v for k, v in reports.items() if not v["ok"]}
    assert not bad, bad
    # the planted values did reach the outputs (the oracle has non-finite entries where the
    # plant makes them), except for the saturation case, which must stay finite
    n_nonfinite = sum(int(np.sum(~np.isfinite(a))) for a in (ry, rdx, rdg, rdw))
    assert (n_nonfinite == 0) == (plant == "g_saturated")
    # the checkpointed step gives the same bits as the separate calls
    for a, b, name in zip((y, rstd, dx, dg), ck[:4], ("y", "rstd", "dx", "dg")):
        assert torch.equal(_as_int(a), _as_int(b)), name
    assert gn.gnorm_device_error(reset=True) == 0


def test_saturated_gate_keeps_its_derivative():
    """g >= 2^24 rounds sigmoid(g) to 1 and 1 + g to g in FP32; the gate's derivative there is
    still dy xhat w (the bracket 1 + g (1 - sigmoid) is 1), not 0."""
    M, N = 64, 128
    case = Case(M, N, seed=7)
    g = np.full((M, N), _bits(3.0e7), dtype=np.uint16)
    case.host["g"] = g
    case.g = bits_to_dev(g)
    _, rstd = gn.gnorm_fwd(case.x, case.g, case.w, case.eps)
    _, dg, _ = gn.gnorm_bwd(case.dy, case.x, case.g, case.w, rstd, dw_fp32=True)
    torch.cuda.synchronize()
    _, _, _, rdg = case.oracle_rows()
    assert np.all(np.abs(rdg) > 0)
    rep = bf16_check(dev_to_f64(dg), rdg)
    assert rep["ok"], rep
