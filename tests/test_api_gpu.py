"""C-ABI argument checks and output bounds on the GPU.

Bad arguments must come back as a status code with nothing launched; outputs must be
written exactly inside their extent (guard regions around every output stay intact).
"""
from __future__ import annotations

import ctypes

import pytest
import torch

from gpu_util import Case

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_norm_b200 as gn
    from gated_norm_b200._lib import (GNORM_ERR_ALIAS, GNORM_ERR_ALIGN, GNORM_ERR_ARG,
                                      GNORM_ERR_NULL, GNORM_ERR_SHAPE, GNORM_ERR_WORKSPACE,
                                      GNORM_OK, lib)


def P(t, byte_offset=0):
    return ctypes.c_void_p(t.data_ptr() + byte_offset)


def _fwd(x, g, w, y, r, M, N, eps=1e-6):
    return lib.gnorm_fwd(x, g, w, eps, y, r, M, N, None)


def test_fwd_argument_errors():
    M, N = 64, 128
    c = Case(M, N)
    y = torch.empty_like(c.x)
    r = torch.empty(M, device="cuda")
    assert _fwd(P(c.x), P(c.g), P(c.w), P(y), P(r), M, N) == GNORM_OK
    assert _fwd(None, P(c.g), P(c.w), P(y), P(r), M, N) == GNORM_ERR_NULL
    assert _fwd(P(c.x), P(c.g), P(c.w), P(y), P(r), M, 100) == GNORM_ERR_SHAPE
    assert _fwd(P(c.x), P(c.g), P(c.w), P(y), P(r), -1, N) == GNORM_ERR_SHAPE
    assert _fwd(P(c.x), P(c.g), P(c.w), P(y), P(r), M, 16392) == GNORM_ERR_SHAPE
    assert _fwd(P(c.x), P(c.g), P(c.w), P(y), P(r), M, 0) == GNORM_ERR_SHAPE
    assert _fwd(P(c.x, 2), P(c.g), P(c.w), P(y), P(r), M - 1, N) == GNORM_ERR_ALIGN
    assert _fwd(P(c.x), P(c.g), P(c.w), P(y), P(r, 2), M - 1, N) == GNORM_ERR_ALIGN
    assert _fwd(P(c.x), P(c.g), P(c.w), P(c.x), P(r), M, N) == GNORM_ERR_ALIAS
    assert _fwd(P(c.x), P(c.g), P(c.w), P(c.g, 256), P(r), M - 1, N) == GNORM_ERR_ALIAS
    assert _fwd(P(c.x), P(c.g), P(c.w), P(y), P(y), M, N) == GNORM_ERR_ALIAS
    assert _fwd(P(c.x), P(c.g), P(c.w), P(y), P(r), M, N, eps=-1.0) == GNORM_ERR_ARG
    assert _fwd(P(c.x), P(c.g), P(c.w), P(y), P(r), M, N, eps=float("nan")) == GNORM_ERR_ARG
    torch.cuda.synchronize()
    assert gn.gnorm_device_error(reset=True) == 0


def test_bwd_argument_errors():
    M, N = 64, 128
    c = Case(M, N)
    _, rstd = gn.gnorm_fwd(c.x, c.g, c.w, 1e-6)
    dx, dg = torch.empty_like(c.x), torch.empty_like(c.x)
    dw = torch.empty(N, dtype=torch.float32, device="cuda")
    need = gn.gnorm_bwd_workspace_bytes(M, N, True)
    ws = torch.zeros(need + 4096, dtype=torch.uint8, device="cuda")

    def call(dy=P(c.dy), x=P(c.x), dxp=P(dx), dwp=P(dw), wsp=P(ws), wsb=need, n=N):
        return lib.gnorm_bwd(dy, x, P(c.g), P(c.w), P(rstd), dxp, P(dg), dwp, 1, 1, M, n, wsp,
                             wsb, None)

    assert call() == GNORM_OK
    assert call(dy=None) == GNORM_ERR_NULL
    assert call(dwp=None) == GNORM_ERR_NULL
    assert call(wsp=None) == GNORM_ERR_WORKSPACE
    assert call(wsb=need - 1) == GNORM_ERR_WORKSPACE
    assert call(wsp=P(ws, 16)) == GNORM_ERR_WORKSPACE
    assert call(dxp=P(c.dy)) == GNORM_ERR_ALIAS          # dx = dy
    assert call(dwp=P(dx, 64)) == GNORM_ERR_ALIAS        # dw inside dx
    assert call(wsp=P(dx)) == GNORM_ERR_ALIAS            # workspace over an output
    assert call(dwp=P(dw, 4)) == GNORM_ERR_ALIGN
    assert call(n=12) == GNORM_ERR_SHAPE
    torch.cuda.synchronize()
    assert gn.gnorm_device_error(reset=True) == 0


def _guarded(n_elems, dtype, guard=4096):
    buf = torch.empty(n_elems + 2 * guard, dtype=dtype, device="cuda")
    pat = torch.tensor(-12345.0, dtype=dtype) if dtype.is_floating_point else 0x5A
    buf.fill_(pat)
    return buf, buf[guard:guard + n_elems], guard


def _guards_intact(buf, guard, n_elems, dtype):
    pat = torch.tensor(-12345.0, dtype=dtype, device="cuda")
    return bool(torch.all(buf[:guard] == pat)) and bool(torch.all(buf[guard + n_elems:] == pat))


@pytest.mark.parametrize("M,N", [(1, 8), (3, 136), (257, 128), (5, 4104), (2, 16384)])
@pytest.mark.parametrize("det", [True, False])
def test_outputs_stay_in_bounds(M, N, det):
    c = Case(M, N, seed=2)
    by, y, gy = _guarded(M * N, torch.bfloat16)
    br, r, gr = _guarded(M, torch.float32)
    bdx, dx, gdx = _guarded(M * N, torch.bfloat16)
    bdg, dg, gdg = _guarded(M * N, torch.bfloat16)
    bdw, dw, gdw = _guarded(N, torch.float32)
    gn.gnorm_ckpt_step(c.x, c.g, c.w, 1e-6, c.dy, y=y.view(M, N), rstd=r, dx=dx.view(M, N),
                       dg=dg.view(M, N), dw=dw, dw_fp32=True, deterministic=det)
    torch.cuda.synchronize()
    assert _guards_intact(by, gy, M * N, torch.bfloat16)
    assert _guards_intact(br, gr, M, torch.float32)
    assert _guards_intact(bdx, gdx, M * N, torch.bfloat16)
    assert _guards_intact(bdg, gdg, M * N, torch.bfloat16)
    assert _guards_intact(bdw, gdw, N, torch.float32)
    assert torch.all(torch.isfinite(y.float())) and torch.all(torch.isfinite(dx.float()))
    assert gn.gnorm_device_error(reset=True) == 0


def test_workspace_query_matches_device():
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for (M, N, det) in [(65536, 128, True), (16384, 4096, False), (7, 8, True)]:
        assert gn.gnorm_bwd_workspace_bytes(M, N, det) == \
            gn.gnorm_bwd_workspace_bytes_for(M, N, det, sms)
