"""The multi-rank path on the CPU: two gloo ranks in spawned processes.

Covers the benchmark's rank environment, max-over-ranks timing and whole-job throughput,
and the rank-ordered gather of per-rank FP32 dw used by the deterministic data-parallel
combine.  (The combine's fixed-order sum runs in the CUDA library and is tested on a GPU.)
"""
from __future__ import annotations

import os
import socket

import torch.multiprocessing as mp

import dist_workers


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_bench_multi_rank_bookkeeping(tmp_path):
    mp.spawn(dist_workers.bench_timing_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2,
             join=True)
    vals = [open(tmp_path / f"rank{r}.txt").read().split() for r in range(2)]
    for mx, value in vals:
        assert float(mx) == 20.0
        # 2 ranks x 100 steps x 1 GB over the slowest rank's 20 ms
        assert abs(float(value) - 2 * 100 * 1e9 / 0.020 / 1e9) < 1e-6


def test_gather_dw_rank_order(tmp_path):
    mp.spawn(dist_workers.gather_dw_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2,
             join=True)
    assert all(os.path.exists(tmp_path / f"gather{r}.ok") for r in range(2))
