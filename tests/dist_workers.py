"""Worker functions for the world-size-2 gloo tests (run in spawned processes)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _setup(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)


def bench_timing_worker(rank, world, port, outdir):
    """The benchmark's multi-rank bookkeeping over gloo: rank env, max over ranks, value."""
    _setup(rank, world, port)
    import torch

    import bench
    r, w, local = bench.dist_env()
    assert (r, w, local) == (rank, world, rank)
    dist = bench.init_dist(torch.device("cpu"), backend="gloo")
    try:
        my_ms = 10.0 * (rank + 1)
        mx = bench.max_over_ranks(my_ms, world, torch.device("cpu"))
        value = bench.whole_job_gbs(1e9, 100, world, mx)
        dist.barrier()
        with open(os.path.join(outdir, f"rank{rank}.txt"), "w") as f:
            f.write(f"{mx} {value}\n")
    finally:
        dist.destroy_process_group()


def gather_dw_worker(rank, world, port, outdir):
    """gated_norm_b200.dp.gather_dw stacks every rank's FP32 dw in rank order."""
    _setup(rank, world, port)
    import torch
    import torch.distributed as dist

    from gated_norm_b200.dp import gather_dw
    dist.init_process_group("gloo")
    try:
        N = 24
        local = torch.arange(N, dtype=torch.float32) + 1000.0 * rank
        parts = gather_dw(local)
        assert parts.shape == (world, N)
        for q in range(world):
            assert torch.equal(parts[q], torch.arange(N, dtype=torch.float32) + 1000.0 * q)
        with open(os.path.join(outdir, f"gather{rank}.ok"), "w") as f:
            f.write("ok\n")
    finally:
        dist.destroy_process_group()
