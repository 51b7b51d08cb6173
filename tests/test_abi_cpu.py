"""The C-ABI library on the CPU: it loads, exports every declared symbol, and its host-only
logic (argument checks that precede any CUDA call, the dispatch rule, workspace sizes)
behaves as specified.  No GPU is needed and no kernel is launched.
"""
from __future__ import annotations

import ctypes
import os
import re
import subprocess

import pytest

import gated_norm_b200 as gn
from gated_norm_b200._lib import (GNORM_ERR_ARG, GNORM_ERR_NULL, GNORM_ERR_SHAPE, LIB_PATH,
                                  SIGNATURES, lib)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gnorm.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GNORM_API\s+[\w\s\*]+?\b(gnorm_\w+)\s*\(", text)))


def test_header_declares_the_api():
    syms = declared_symbols()
    for s in ("gnorm_fwd", "gnorm_bwd", "gnorm_ckpt_step", "gnorm_bwd_workspace_bytes",
              "gnorm_status_string", "gnorm_plan_query"):
        assert s in syms


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (gnorm_\w+)", out))
    assert set(declared_symbols()) <= exported
    assert set(SIGNATURES) == set(declared_symbols())
    for s in declared_symbols():
        assert hasattr(lib, s)
    # nothing else leaks: the statically linked CUDA runtime stays hidden
    assert not re.search(r"\bT cuda\w+", out)


def test_status_strings():
    for code in range(0, -9, -1):
        s = gn.gnorm_status_string(code)
        assert s.startswith("GNORM_")
    assert "unknown" in gn.gnorm_status_string(-99)


def test_build_info():
    assert "sm_100a" in gn.gnorm_build_info()


def test_host_checks_precede_cuda():
    """These fail on argument checks, before any CUDA call, so they run without a GPU."""
    p = ctypes.c_void_p(4096)
    assert lib.gnorm_fwd(None, p, p, 1e-6, p, p, 4, 128, None) == GNORM_ERR_NULL
    assert lib.gnorm_fwd(p, p, p, 1e-6, p, p, 4, 100, None) == GNORM_ERR_SHAPE
    assert lib.gnorm_fwd(p, p, p, -1.0, p, p, 4, 128, None) == GNORM_ERR_ARG
    assert lib.gnorm_fwd(None, None, None, 1e-6, None, None, 0, 128, None) == 0  # M = 0: no-op
    assert lib.gnorm_bwd(p, p, p, p, p, p, p, None, 0, 1, 4, 128, p, 1 << 20, None) == \
        GNORM_ERR_NULL
    assert lib.gnorm_ckpt_step(p, p, p, 1e-6, p, p, p, p, p, p, 0, 1, 4, 7, p, 1 << 20, None) == \
        GNORM_ERR_SHAPE


# ------------------------------------------------------------------------- dispatch rule

SM_COUNTS = (148, 132, 212)
NS = (8, 16, 32, 64, 120, 128, 136, 256, 264, 512, 1000, 1024, 2048, 4096, 4104, 8192, 16384)
MS = (1, 2, 7, 100, 147, 148, 149, 1024, 4733, 65536, 368640, 1 << 22)


@pytest.mark.parametrize("sms", SM_COUNTS)
@pytest.mark.parametrize("kind", [0, 1])
def test_plan_invariants(sms, kind):
    for N in NS:
        for M in MS:
            for det in (True, False):
                p = gn.gnorm_plan_query(kind, M, N, det, sms)
                R, G = p["rows_per_stage"], p["grid"]
                assert 1 <= R and p["stages"] >= 2
                assert p["num_blocks"] * R >= M and (p["num_blocks"] - 1) * R < M
                assert 1 <= G <= sms * p["ctas_per_sm"] and G <= p["num_blocks"]
                assert p["threads_per_row"] * p["chunks_per_thread"] * 8 >= N
                assert p["consumer_threads"] % p["threads_per_row"] == 0
                assert p["consumer_threads"] + 32 <= 1024
                tensors = 2 if kind == 0 else 3
                stage = -(-tensors * R * N * 2 // 128) * 128
                assert p["smem_bytes"] >= 1024 + p["stages"] * stage
                assert p["smem_bytes"] <= 232448
                # static round-robin: no CTA gets more than one block above the mean
                per_cta = -(-p["num_blocks"] // G)
                assert per_cta * R - M / G < R + 1
                if kind == 1:
                    groups = p["consumer_threads"] // p["threads_per_row"]
                    assert p["smem_bytes"] >= 1024 + groups * N * 4 + p["consumer_threads"] * 16
                    assert p["partials"] == G
                    assert p["dynamic_schedule"] == (0 if det else 1)
                    if det:
                        assert p["fused_reduce"] == 0


def test_plan_is_a_pure_function():
    a = gn.gnorm_plan_query(1, 368640, 128, True, 148)
    b = gn.gnorm_plan_query(1, 368640, 128, True, 148)
    assert a == b


def test_tier_edge_rows_per_sm():
    """Latency tier (one block per CTA) up to the stage's target rows per SM, then the
    streaming tier (several equal blocks per CTA) -- tested on both sides of the edge."""
    for sms in SM_COUNTS:
        edge = None
        for rows_per_sm in range(1, 200):
            p = gn.gnorm_plan_query(0, rows_per_sm * sms, 128, True, sms)
            if p["num_blocks"] > p["grid"]:
                edge = rows_per_sm
                break
        assert edge is not None
        below = gn.gnorm_plan_query(0, (edge - 1) * sms, 128, True, sms)
        above = gn.gnorm_plan_query(0, edge * sms, 128, True, sms)
        assert below["num_blocks"] == below["grid"] == sms
        assert above["num_blocks"] > above["grid"]
        assert above["rows_per_stage"] * 2 >= below["rows_per_stage"]


def test_plan_errors():
    with pytest.raises(gn.GnormError):
        gn.gnorm_plan_query(0, 10, 12, True, 148)
    with pytest.raises(gn.GnormError):
        gn.gnorm_plan_query(2, 10, 128, True, 148)
    with pytest.raises(gn.GnormError):
        gn.gnorm_plan_query(0, 10, 128, True, 0)
    with pytest.raises(gn.GnormError):  # shared memory too small for two stages of a row
        gn.gnorm_plan_query(1, 10, 16384, True, 148, smem_per_block=64 * 1024)


def test_workspace_bytes():
    for sms in SM_COUNTS:
        for N in (128, 4096):
            b = gn.gnorm_bwd_workspace_bytes_for(65536, N, True, sms)
            p = gn.gnorm_plan_query(1, 65536, N, True, sms)
            assert b % 256 == 0
            assert b >= 256 + p["partials"] * N * 4
    assert gn.gnorm_bwd_workspace_bytes_for(10, 12, True, 148) == 0


def test_tuning_knobs_change_plans_and_reset():
    base = gn.gnorm_plan_query(0, 1 << 20, 128, True, 148)
    try:
        gn.gnorm_set_tuning(stage_bytes=8192, max_stages=4)
        p = gn.gnorm_plan_query(0, 1 << 20, 128, True, 148)
        assert p["stages"] <= 4 and p["rows_per_stage"] < base["rows_per_stage"]
    finally:
        gn.gnorm_set_tuning()
    assert gn.gnorm_plan_query(0, 1 << 20, 128, True, 148) == base
