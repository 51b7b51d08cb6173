"""Host logic of bench.py that needs no GPU: the source digest that ties a committed ncu
summary under profiles/ to the kernel sources it was captured from."""
from __future__ import annotations

import os
import shutil

import bench

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "gated_norm_b200", "csrc")


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
