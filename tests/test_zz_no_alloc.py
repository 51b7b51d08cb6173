"""gnorm_bwd_noalloc: the backward for callers that cannot allocate device memory (GPU).

Such callers -- a runtime whose device memory another allocator owns up front, a
latency-critical loop that must not hit cudaMalloc's implicit synchronisation, a plug-in
that only receives tensors -- cannot hand gnorm_bwd a workspace.  gnorm_bwd_noalloc keeps
its scratch in a static device array inside the library instead.  This file checks,
through the C ABI, on two calls in a row: in deterministic mode the results are bitwise
those of gnorm_bwd (the same plan and kernels); in either mode dx and dg are bitwise those
of gnorm_bwd and dw is within the dw tolerance of gnorm_bwd's; and all three are within the
tolerances of the FP64 oracle.  Sizes beyond the array's limit are refused.

It is named so that pytest collects it last; it passes alone in a fresh process and after
the other tests.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

from gpu_util import Case, dev_to_f64, sample_rows
from tolerance import bf16_check, dw_fp32_check

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_norm_b200 as gn
    from gated_norm_b200._lib import GNORM_ERR_UNSUPPORTED, GNORM_OK, lib


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc(case, rstd, dx, dg, dw, dw_fp32, det, stream):
    return lib.gnorm_bwd_noalloc(_p(case.dy), _p(case.x), _p(case.g), _p(case.w), _p(rstd),
                                 _p(dx), _p(dg), _p(dw), int(dw_fp32), int(det), case.M, case.N,
                                 ctypes.c_void_p(stream.cuda_stream))


def _dw_check(got, ref, dw_fp32):
    return dw_fp32_check(got, ref) if dw_fp32 else bf16_check(got, ref)


@pytest.mark.parametrize("M,N", [(65536, 128), (1537, 136), (16384, 4096), (3, 8)])
@pytest.mark.parametrize("det", [True, False])
@pytest.mark.parametrize("dw_fp32", [True, False])
def test_noalloc_matches_workspace_backward(M, N, det, dw_fp32):
    case = Case(M, N, seed=17)
    stream = torch.cuda.current_stream()
    _, rstd = gn.gnorm_fwd(case.x, case.g, case.w, case.eps)
    ref_dx, ref_dg, ref_dw = gn.gnorm_bwd(case.dy, case.x, case.g, case.w, rstd,
                                          dw_fp32=dw_fp32, deterministic=det)
    torch.cuda.synchronize()
    rows = sample_rows(M, n_random=512) if M * N > (1 << 22) else None
    _, _, o_dx, o_dg = case.oracle_rows(rows, rstd=dev_to_f64(rstd) if rows is None
                                        else dev_to_f64(rstd)[rows])
    o_dw = case.oracle_dw()
    for _ in range(2):  # two calls in a row share (and must re-clear) the static scratch
        dx, dg = torch.empty_like(case.x), torch.empty_like(case.x)
        dw = torch.empty(N, dtype=torch.float32 if dw_fp32 else torch.bfloat16, device="cuda")
        assert _noalloc(case, rstd, dx, dg, dw, dw_fp32, det, stream) == GNORM_OK
        torch.cuda.synchronize()
        # dx and dg do not depend on the mode or the scratch: bitwise those of gnorm_bwd
        assert torch.equal(dx, ref_dx) and torch.equal(dg, ref_dg)
        if det:
            assert torch.equal(dw, ref_dw)  # same plan, same kernels, fixed order
        else:
            rep = _dw_check(dev_to_f64(dw), dev_to_f64(ref_dw), dw_fp32)
            assert rep["ok"], rep
        sel = (lambda a: a) if rows is None else (lambda a: a[rows])
        for got, ref, name in ((sel(dev_to_f64(dx)), o_dx, "dx"), (sel(dev_to_f64(dg)), o_dg, "dg")):
            rep = bf16_check(got, ref)
            assert rep["ok"], (name, rep)
        rep = _dw_check(dev_to_f64(dw), o_dw, dw_fp32)
        assert rep["ok"], ("dw vs oracle", rep)
    assert gn.gnorm_device_error(reset=True) == 0


def test_noalloc_refuses_sizes_beyond_its_scratch():
    case = Case(2048, 16384, seed=1)  # partials x 16384 x 4 bytes exceed the 4 MiB array
    _, rstd = gn.gnorm_fwd(case.x, case.g, case.w, case.eps)
    dx, dg = torch.empty_like(case.x), torch.empty_like(case.x)
    dw = torch.empty(case.N, dtype=torch.float32, device="cuda")
    st = _noalloc(case, rstd, dx, dg, dw, True, True, torch.cuda.current_stream())
    assert st == GNORM_ERR_UNSUPPORTED
    assert "GNORM_ERR_UNSUPPORTED" in gn.gnorm_status_string(st)
