"""Host logic of bench.py that needs no GPU: the source digest that ties a committed ncu
summary under profiles/ to the kernel sources it was captured from."""
from __future__ import annotations

import os
import shutil

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "gated_norm_b200", "csrc")


def _copy(tmp_path):
    dst = tmp_path / "csrc"
    shutil.copytree(CSRC, dst)
    return dst


def test_digest_ignores_comments_only(tmp_path):
    d = _copy(tmp_path)
    base = bench.source_digest(str(d))
    assert base == bench.source_digest()
    p = d / "device_common.cuh"
    text = p.read_text()
    # a new line comment, a new block comment and an edited comment keep the digest
    p.write_text("// a note\n" + text.replace("#pragma once", "#pragma once  /* x */", 1))
    assert bench.source_digest(str(d)) == base
    # a code change does not
    p.write_text(text.replace("#pragma once", "#pragma once\nstatic int gnorm_probe_ = 1;", 1))
    assert bench.source_digest(str(d)) != base


def test_digest_excludes_host_only_files(tmp_path):
    d = _copy(tmp_path)
    base = bench.source_digest(str(d))
    for name in bench._DIGEST_EXCLUDED:
        with open(d / name, "a") as f:
            f.write("\nstatic int gnorm_host_only_ = 0;\n")
    assert bench.source_digest(str(d)) == base


def test_profiles_match_the_sources():
    """The committed traffic summaries of the default workload were captured from these
    sources, so bench.py reports their traffic instead of null."""
    for kernel in ("fwd", "bwd", "fwd_bwd"):
        assert bench.profiled_traffic(f"{kernel}_kernel", "mid_262144x256") is not None, kernel


def _run_bench(*args):
    import subprocess
    import sys

    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                          capture_output=True, text=True, timeout=300, cwd=ROOT)


def test_reference_arm_prints_one_json_line():
    """`bench.py --impl reference`: the FP64 oracle timed on the host cores, one JSON line
    with the arm's keys (the same metric, unit and workload as the CUDA arm)."""
    import json

    res = _run_bench("--impl", "reference", "--steps", "2", "--warmup", "3",
                     "--workload", "small_1024x128", "--ref-seconds", "2")
    assert res.returncode == 0, res.stderr
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["higher_is_better"] is True
    assert d["unit"] == "GB/s" and d["value"] > 0 and d["steps"] == 2
    assert d["config"]["workload"] == "small_1024x128"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_cuda_arm_fails_loudly_without_a_gpu():
    """No CPU fallback: without a CUDA device the CUDA arm exits with an error."""
    import torch

    if torch.cuda.is_available():
        return
    res = _run_bench("--steps", "3", "--warmup", "3", "--no-per-config")
    assert res.returncode != 0
    assert "no CUDA device" in (res.stderr + res.stdout)


def test_warmup_below_three_is_rejected():
    res = _run_bench("--warmup", "1")
    assert res.returncode != 0 and "at least 3" in res.stderr
