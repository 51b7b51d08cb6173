"""gnorm_ckpt_step_host: the checkpointed step on host buffers, chunked and pipelined (GPU).

Rows are independent, so y, rstd, dx and dg must equal the device entry point's bit for bit
whatever the chunking; dw is a fixed-order sum of per-chunk FP32 rows, so it must be within
its tolerance of the FP64 oracle, bitwise stable from call to call in deterministic mode,
and bitwise equal to the device entry point's when there is one chunk.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from gpu_util import Case, dev_to_f64
from tolerance import bf16_check, dw_fp32_check

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_norm_b200 as gn


def host_inputs(case: Case, pin: bool = True):
    def cpu(bits):
        t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
        return t.pin_memory() if pin else t.clone()
    return tuple(cpu(case.host[k]) for k in ("x", "g", "w", "dy"))


def run_host(case, *, dw_fp32, det, pin=True, chunk_rows=None):
    x, g, w, dy = host_inputs(case, pin)
    try:
        if chunk_rows is not None:
            gn.gnorm_set_tuning(host_chunk_bytes=6 * case.N * chunk_rows)
        out = gn.gnorm_ckpt_step_host(x, g, w, case.eps, dy, dw_fp32=dw_fp32,
                                      deterministic=det)
        torch.cuda.synchronize()
    finally:
        gn.gnorm_set_tuning()
    return out


def check_dw(dw, case):
    ref = case.oracle_dw()
    got = dev_to_f64(dw)
    rep = dw_fp32_check(got, ref) if dw.dtype == torch.float32 else bf16_check(got, ref)
    assert rep["ok"], rep


# (M, N, rows per chunk or None for the built-in chunk size)
CASES = [
    (1024, 128, None),   # one chunk: everything equals the device entry point
    (1037, 128, 100),    # 11 chunks, ragged last chunk of 37 rows
    (700, 4096, 64),     # wide rows, 11 chunks
    (513, 256, 1),       # one row per chunk: 256 chunks plus one more row each
    (3, 16, None),
]


@pytest.mark.parametrize("M,N,chunk_rows", CASES)
@pytest.mark.parametrize("dw_fp32", [True, False])
def test_host_step_matches_device_step(M, N, chunk_rows, dw_fp32):
    case = Case(M, N, seed=31)
    ref = gn.gnorm_ckpt_step(case.x, case.g, case.w, case.eps, case.dy, dw_fp32=dw_fp32,
                             deterministic=True)
    torch.cuda.synchronize()
    out = run_host(case, dw_fp32=dw_fp32, det=True, chunk_rows=chunk_rows)
    for a, b, name in zip(ref[:4], out[:4], ("y", "rstd", "dx", "dg")):
        assert torch.equal(a.cpu(), b), name
    rows = chunk_rows if chunk_rows is not None else M
    chunks = -(-M // max(1, min(rows, M)))
    if chunks > 256:  # the library caps the number of chunks
        chunks = 256
    if chunks == 1:
        assert torch.equal(ref[4].cpu(), out[4])
    check_dw(out[4], case)
    again = run_host(case, dw_fp32=dw_fp32, det=True, chunk_rows=chunk_rows)
    for a, b in zip(out, again):
        assert torch.equal(a, b)
    assert gn.gnorm_device_error(reset=True) == 0


def test_host_step_nondeterministic_and_pageable():
    case = Case(2049, 128, seed=5)
    det = run_host(case, dw_fp32=True, det=True, chunk_rows=300)
    nd = run_host(case, dw_fp32=True, det=False, chunk_rows=300)
    page = run_host(case, dw_fp32=True, det=True, pin=False, chunk_rows=300)
    for a, b, c in zip(det[:4], nd[:4], page[:4]):
        assert torch.equal(a, b) and torch.equal(a, c)
    assert torch.equal(det[4], page[4])
    check_dw(nd[4], case)


def test_host_step_zero_rows_and_errors():
    N = 128
    x = torch.empty((0, N), dtype=torch.bfloat16)
    w = torch.ones(N, dtype=torch.bfloat16)
    dw = torch.full((N,), 7.0)
    out = gn.gnorm_ckpt_step_host(x, x, w, 1e-6, x, dw=dw, dw_fp32=True)
    torch.cuda.synchronize()
    assert torch.equal(out[4], torch.zeros(N))

    case = Case(64, N, seed=2)
    hx, hg, hw, hdy = host_inputs(case)
    need = gn.gnorm_ckpt_step_host_bytes(64, N, True)
    assert need > 0
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(gn.GnormError) as e:
        gn.gnorm_ckpt_step_host(hx, hg, hw, 1e-6, hdy, dev_buf=small)
    assert e.value.status == -6  # GNORM_ERR_WORKSPACE
    y = torch.empty((64, N), dtype=torch.bfloat16).pin_memory()
    with pytest.raises(gn.GnormError) as e:
        gn.gnorm_ckpt_step_host(hx, hg, hw, 1e-6, hdy, y=y, dx=y)
    assert e.value.status == -4  # GNORM_ERR_ALIAS
    with pytest.raises(gn.GnormError) as e:
        gn.gnorm_ckpt_step_host(hx, hg, hw, float("nan"), hdy)
    assert e.value.status == -8  # GNORM_ERR_ARG
    torch.cuda.synchronize()
    assert gn.gnorm_device_error(reset=True) == 0
