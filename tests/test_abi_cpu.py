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
import torch

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
    waited = ctypes.c_ulonglong(0)
    assert lib.gnorm_selftest_wait_timeout(0, ctypes.byref(waited)) == GNORM_ERR_ARG
    assert lib.gnorm_selftest_wait_timeout(1000, None) == GNORM_ERR_NULL


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
                rows_per_sm = -(-M // sms)
                if kind == 0:
                    direct = N <= 256 and rows_per_sm * 4 * N < 512 * 1024
                else:
                    direct = N <= 256 and rows_per_sm * 6 * N < 256 * 1024
                assert p["direct_loads"] == direct
                if p["direct_loads"]:  # rows straight into registers, no stages
                    tpr = p["threads_per_row"]
                    ctas = 4 if kind == 0 else 2
                    assert p["chunks_per_thread"] == 1 and tpr * 8 >= N and tpr <= 32
                    assert p["consumer_threads"] == 256 and R == (256 // tpr) * 2
                    assert p["stages"] == 0 and p["smem_bytes"] == 0
                    assert p["num_blocks"] * R >= M and (p["num_blocks"] - 1) * R < M
                    assert 1 <= G <= min(p["num_blocks"], ctas * sms)
                    assert p["ctas_per_sm"] == ctas
                    if kind == 1:  # static rows in both modes; one partial row per CTA
                        assert p["partials"] == G and p["dynamic_schedule"] == 0
                        assert p["fused_reduce"] == 0
                    continue
                assert 1 <= R and p["stages"] >= 2
                assert p["num_blocks"] * R >= M and (p["num_blocks"] - 1) * R < M
                assert 1 <= G <= sms * p["ctas_per_sm"] and G <= p["num_blocks"]
                assert p["threads_per_row"] * p["chunks_per_thread"] * 8 >= N
                assert p["consumer_threads"] % p["threads_per_row"] == 0
                assert p["consumer_threads"] + 32 <= 1024
                if kind == 1 and p["threads_per_row"] <= 16 and p["chunks_per_thread"] == 1:
                    assert p["consumer_threads"] == 512
                tensors = 2 if kind == 0 else 3
                tensor = -(-(R * N * 2) // 128) * 128
                stage = -(-(tensors * tensor + (4 * R if kind == 1 else 0)) // 128) * 128
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
                    assert p["fused_reduce"] == 0  # second launch unless the knob asks


def test_plan_is_a_pure_function():
    a = gn.gnorm_plan_query(1, 368640, 128, True, 148)
    b = gn.gnorm_plan_query(1, 368640, 128, True, 148)
    assert a == b


def test_tier_edge_rows_per_sm():
    """The rows-per-SM tiers, each tested on both sides of its edge.

    Forward: under 512 KB of staged rows (x and g) per SM the latency tier runs 3 CTAs
    per SM with small stages, from there on the streaming tier runs 2.  Within a tier,
    one block per CTA while the CTA's rows fit one stage, then equal multi-block shares."""
    for sms in SM_COUNTS:
        N = 128
        rows_edge = 512 * 1024 // (4 * N)  # rows per SM where the staged bytes reach 512 KB
        lat = gn.gnorm_plan_query(0, (rows_edge - 1) * sms, N, True, sms)
        stream = gn.gnorm_plan_query(0, rows_edge * sms, N, True, sms)
        # narrow rows in the latency tier: loaded straight into registers, 4 CTAs per SM
        assert lat["direct_loads"] == 1 and lat["ctas_per_sm"] == 4 and lat["stages"] == 0
        assert stream["direct_loads"] == 0 and stream["ctas_per_sm"] == 2
        try:  # with staging forced, the latency tier stages ~16 KB with 3 CTAs per SM where
            # the geometry's registers allow it (one chunk per thread), else 2
            gn.gnorm_set_tuning(fwd_direct=2)
            lat = gn.gnorm_plan_query(0, (rows_edge - 1) * sms, N, True, sms)
            assert lat["direct_loads"] == 0
            assert lat["ctas_per_sm"] == (3 if lat["chunks_per_thread"] == 1 else 2)
            assert lat["rows_per_stage"] * 4 * N <= 16384 < stream["rows_per_stage"] * 4 * N
            gn.gnorm_set_tuning(fwd_direct=1)  # and loads straight into registers at any size
            assert gn.gnorm_plan_query(0, rows_edge * sms, N, True, sms)["direct_loads"] == 1
            assert gn.gnorm_plan_query(0, rows_edge * sms, 264, True, sms)["direct_loads"] == 0
        finally:
            gn.gnorm_set_tuning()
        # the wide-row forward uses the same byte rule; its registers cap it at 2 CTAs per SM
        wide_lat = gn.gnorm_plan_query(0, 8 * sms, 4096, True, sms)
        wide_stream = gn.gnorm_plan_query(0, 64 * sms, 4096, True, sms)
        assert wide_lat["ctas_per_sm"] == wide_stream["ctas_per_sm"] == 2
        assert wide_lat["rows_per_stage"] == 1 and wide_stream["rows_per_stage"] == 3
        try:
            gn.gnorm_set_tuning(fwd_direct=2, bwd_direct=2)  # the staged kernels' blocks
            for kind in (0, 1):
                big = gn.gnorm_plan_query(kind, 1 << 12, N, True, sms)
                ctas = sms * big["ctas_per_sm"]
                edge = None
                for rows_per_cta in range(1, 400):
                    p = gn.gnorm_plan_query(kind, rows_per_cta * ctas, N, True, sms)
                    if p["ctas_per_sm"] != big["ctas_per_sm"]:
                        break
                    if p["num_blocks"] > p["grid"]:
                        edge = rows_per_cta
                        break
                if edge is None:
                    continue
                below = gn.gnorm_plan_query(kind, (edge - 1) * ctas, N, True, sms)
                above = gn.gnorm_plan_query(kind, edge * ctas, N, True, sms)
                assert below["num_blocks"] == below["grid"] == ctas
                assert below["rows_per_stage"] == edge - 1
                assert above["num_blocks"] > above["grid"]
        finally:
            gn.gnorm_set_tuning()


def test_ctas_per_sm_never_exceeds_the_compiled_residency():
    for kind in (0, 1):
        for N in NS:
            for M in MS:
                for knob in (0, 2, 3, 4):
                    try:
                        gn.gnorm_set_tuning(ctas_per_sm=knob)
                        p = gn.gnorm_plan_query(kind, M, N, True, 148)
                    finally:
                        gn.gnorm_set_tuning()
                    tpr, cpt = p["threads_per_row"], p["chunks_per_thread"]
                    fit = 1 if p["consumer_threads"] > 256 else (
                        (3 if cpt == 1 else 2 if cpt <= 4 else 1) if kind == 0 else
                        (2 if cpt == 1 else 1))
                    if p["direct_loads"]:  # the direct-load kernels' compiled residency
                        fit = 4 if kind == 0 else 2
                    assert p["ctas_per_sm"] <= fit


def test_plan_errors():
    with pytest.raises(gn.GnormError):
        gn.gnorm_plan_query(0, 10, 12, True, 148)
    with pytest.raises(gn.GnormError):  # kinds are 0 (forward), 1 (backward), 2 (fused)
        gn.gnorm_plan_query(3, 10, 128, True, 148)
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


def test_forced_geometry_knob():
    try:
        gn.gnorm_set_tuning(threads_per_row=256, chunks_per_thread=2)
        p = gn.gnorm_plan_query(0, 4096, 4096, True, 148)
        assert (p["threads_per_row"], p["chunks_per_thread"]) == (256, 2)
        with pytest.raises(gn.GnormError):  # 256 x 2 x 8 < 8192 columns
            gn.gnorm_plan_query(0, 4096, 8192, True, 148)
        gn.gnorm_set_tuning(threads_per_row=64, chunks_per_thread=8)
        assert gn.gnorm_plan_query(0, 64, 4096, True, 148)["threads_per_row"] == 64
        with pytest.raises(gn.GnormError):  # forward-only geometry
            gn.gnorm_plan_query(1, 64, 4096, True, 148)
        gn.gnorm_set_tuning(threads_per_row=48, chunks_per_thread=3)
        with pytest.raises(gn.GnormError):  # not compiled
            gn.gnorm_plan_query(0, 64, 128, True, 148)
    finally:
        gn.gnorm_set_tuning()


def test_tail_and_l2_knobs_in_plans():
    base = gn.gnorm_plan_query(1, 65536, 128, True, 148)
    assert base["fused_reduce"] == 0 and base["l2_prefetch"] == 0
    try:
        gn.gnorm_set_tuning(tail_reduce=1, l2_prefetch=1)
        p = gn.gnorm_plan_query(1, 65536, 128, True, 148)
        assert p["fused_reduce"] == 1 and p["l2_prefetch"] == 1
        gn.gnorm_set_tuning(tail_reduce=1)
        assert gn.gnorm_plan_query(1, 65536, 4096, True, 148)["fused_reduce"] == 0  # too big
        with pytest.raises(TypeError):
            gn.gnorm_set_tuning(no_such_knob=1)
    finally:
        gn.gnorm_set_tuning()
    assert gn.gnorm_plan_query(1, 65536, 128, True, 148) == base


# ------------------------------------------------------------ strided rows (host checks)

def _fwd_desc(**kw):
    from gated_norm_b200._lib import GnormFwdDesc
    base = dict(x=1 << 20, ldx=0, g=2 << 20, ldg=0, w=3 << 20, w_fp32=0, eps=1e-6,
                y=4 << 20, ldy=0, rstd=5 << 20, M=4, N=128)
    base.update(kw)
    return GnormFwdDesc(**base)


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="fake pointers that pass the host checks would reach a launch")
def test_strided_descriptor_checks_precede_cuda():
    """Stride and alias rules are host checks; a descriptor that passes them goes on to the
    device query, which fails without a GPU (GNORM_ERR_CUDA), so the two are told apart."""
    from gated_norm_b200._lib import (GNORM_ERR_ALIAS, GNORM_ERR_ALIGN, GNORM_ERR_CUDA,
                                      GNORM_ERR_SHAPE)
    fwd = lambda **kw: lib.gnorm_fwd_ex(ctypes.byref(_fwd_desc(**kw)), None)
    assert fwd(ldx=100) == GNORM_ERR_SHAPE            # stride shorter than a row
    assert fwd(ldx=132) == GNORM_ERR_ALIGN            # rows would not start 16-byte aligned
    base = 1 << 24
    # x and g as the two column halves of one [M, 256] buffer (inputs may share memory)
    assert fwd(x=base, ldx=256, g=base + 256, ldg=256) == GNORM_ERR_CUDA
    # y in the other half of x's buffer: no element shared -> passes the alias check
    assert fwd(x=base, ldx=256, y=base + 256, ldy=256) == GNORM_ERR_CUDA
    # y shifted by 8 columns into x's rows: shares elements -> rejected
    assert fwd(x=base, ldx=256, y=base + 16, ldy=256) == GNORM_ERR_ALIAS
    # y one whole row below x with the same stride: rows overlap -> rejected
    assert fwd(x=base, ldx=256, y=base + 512, ldy=256) == GNORM_ERR_ALIAS
    # y past the end of x's last row
    assert fwd(x=base, ldx=256, y=base + 4 * 512, ldy=256) == GNORM_ERR_CUDA
    # different strides that interleave: the check is conservative -> rejected
    assert fwd(x=base, ldx=256, y=base + 256, ldy=384) == GNORM_ERR_ALIAS


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="fake pointers that pass the host checks would reach a copy")
def test_host_step_checks_precede_cuda():
    """gnorm_ckpt_step_host checks its arguments before any CUDA call; arguments that pass
    go on to the device query, which fails without a GPU (GNORM_ERR_CUDA)."""
    from gated_norm_b200._lib import GNORM_ERR_ALIAS, GNORM_ERR_CUDA, GNORM_ERR_WORKSPACE

    def call(M=64, N=128, eps=1e-6, dev_buf=1 << 30, **ptrs):
        p = {k: (i + 1) << 26 for i, k in enumerate(("x", "g", "w", "dy", "y", "rstd", "dx",
                                                     "dg", "dw"))}
        p.update(ptrs)
        v = {k: ctypes.c_void_p(a) if a is not None else None for k, a in p.items()}
        return lib.gnorm_ckpt_step_host(v["x"], v["g"], v["w"], eps, v["dy"], v["y"], v["rstd"],
                                        v["dx"], v["dg"], v["dw"], 1, 1, M, N,
                                        ctypes.c_void_p(dev_buf) if dev_buf else None, 1 << 30,
                                        None)
    assert call(N=12) == GNORM_ERR_SHAPE
    assert call(M=-1) == GNORM_ERR_SHAPE
    assert call(eps=float("inf")) == GNORM_ERR_ARG
    assert call(dw=None) == GNORM_ERR_NULL
    assert call(dg=None) == GNORM_ERR_NULL
    assert call(dev_buf=None) == GNORM_ERR_WORKSPACE
    assert call(dev_buf=(1 << 30) + 16) == GNORM_ERR_WORKSPACE  # not 256-byte aligned
    assert call(y=(1 << 26) + 64) == GNORM_ERR_ALIAS            # y inside x
    assert call(dx=(5 << 26) + 4096) == GNORM_ERR_ALIAS         # dx inside y
    assert call() == GNORM_ERR_CUDA                             # passes: device query fails
    assert lib.gnorm_ckpt_step_host_bytes(64, 128, 1) == 0      # no device
    assert lib.gnorm_ckpt_step_host_bytes(64, 12, 1) == 0       # bad shape


def test_ckpt_ex_requires_consistent_descriptors():
    from gated_norm_b200._lib import GNORM_ERR_ARG, GnormBwdDesc
    f = _fwd_desc()
    b = GnormBwdDesc(dy=6 << 20, x=7 << 20, dx=8 << 20, dg=9 << 20, dw=10 << 20, M=4, N=128,
                     workspace=11 << 20, workspace_bytes=1 << 20)
    assert lib.gnorm_ckpt_step_ex(ctypes.byref(f), ctypes.byref(b), None) == GNORM_ERR_ARG
    b.x = f.x
    b.M = 5
    assert lib.gnorm_ckpt_step_ex(ctypes.byref(f), ctypes.byref(b), None) == GNORM_ERR_ARG


def test_header_is_c_and_links_from_c(tmp_path):
    """include/gnorm.h compiles as C99 and a C program links and calls libgnorm."""
    exe = tmp_path / "c_abi_example"
    libdir = os.path.dirname(LIB_PATH)
    src = os.path.join(ROOT, "tests", "c_abi_example.c")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    src, "-o", str(exe), "-L", libdir, "-lgnorm", f"-Wl,-rpath,{libdir}"],
                   check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    fields = dict(kv.split("=") for kv in out.split()[:7])
    p = gn.gnorm_plan_query(1, 368640, 128, True, 148)
    assert int(fields["grid"]) == p["grid"] and int(fields["rows"]) == p["rows_per_stage"]
    assert int(fields["ws"]) == gn.gnorm_bwd_workspace_bytes_for(368640, 128, True, 148)
    assert int(fields["null"]) == GNORM_ERR_NULL and int(fields["shape"]) == GNORM_ERR_SHAPE
    assert "sm_100a" in out


def test_header_states_the_workspace_rule_after_a_timeout():
    """A call whose bounded wait gave up may leave the workspace header nonzero; the header
    tells the caller to zero it again before reuse."""
    text = open(os.path.join(ROOT, "include", "gnorm.h")).read()
    assert "zero the first GNORM_WORKSPACE_ALIGN bytes again" in text
    assert "every call that\n *   completes normally leaves them zero again" in text


def test_fused_plan_is_the_backward_plan_with_its_own_narrow_geometry():
    """Kind 2 (the forward fused into the backward) plans like the backward -- same CTAs,
    blocks, stages, direct-load decision and partial rows, so the same workspace suffices --
    except that rows of N <= 128 take 8 threads x 2 chunks (16 x 1 in the backward)."""
    for sms in SM_COUNTS:
        for M, N in ((368640, 128), (65536, 128), (4099, 64), (262144, 256), (16384, 4096),
                     (1024, 128), (37, 8200)):
            b = gn.gnorm_plan_query(1, M, N, True, sms)
            f = gn.gnorm_plan_query(2, M, N, True, sms)
            assert f["kind"] == 2
            for k in ("rows_per_stage", "stages", "grid", "num_blocks", "direct_loads",
                      "partials", "dynamic_schedule", "ctas_per_sm"):
                assert f[k] == b[k], (M, N, k)
            if 64 < N <= 128 and not f["direct_loads"]:
                assert (f["threads_per_row"], f["chunks_per_thread"]) == (8, 2)
                assert (b["threads_per_row"], b["chunks_per_thread"]) == (16, 1)
            elif not f["direct_loads"]:
                assert (f["threads_per_row"], f["chunks_per_thread"]) == \
                    (b["threads_per_row"], b["chunks_per_thread"])
