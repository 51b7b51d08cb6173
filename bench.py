"""Benchmark of the SiLU-gated RMSNorm training step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--nondeterministic] [--dw-fp32]

A step is one checkpointed training step over one batch of seeded synthetic rows:
forward, forward again (recompute), backward with the dw reduction -- every stage of the
path -- replayed from one CUDA graph ("ckptg").  Each timed step also replays the backward
("bwdg") and the forward ("fwdg") alone, each from its own graph, for the per-operation
times and the roofline of the dominant kernel (the forward: two launches per step, the
largest share of the step's device time).  The default workload is 65536 x 128 (a
per-head gated norm of a linear-attention output, 512 heads x 128 tokens).  Times are
CUDA-event device times on the launching stream; L2 is flushed (256 MiB write) before
every timed replay, outside the events.  `value` is the checkpointed step's algorithmic
HBM bytes of the whole job / the max-over-ranks summed step time (GB/s).

Under torchrun (N > 1) every rank runs its own batch (weak scaling, no collective on the
data path; the rows of a data-parallel batch are independent).  `--impl reference` times
the FP64 CPU oracle on a bounded sample of the same workload (rank 0 only).  `--floor`
adds, after the timed region, the same measurement of an empty graph and of torch
elementwise kernels that move the forward's and backward's main streams (context for the
fixed per-launch cost at small sizes).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synthetic import WORKLOADS, bf16_bits_to_f64, make_inputs  # noqa: E402

METRIC = "fwd / bwd / ckpt-step µs and achieved HBM GB/s (% of B200 roofline), 1 GPU"
DEFAULT_WORKLOAD = "linattn_65536x128"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20


# ----------------------------------------------------------------------------- bytes

def fwd_bytes(M, N):
    return M * (6 * N + 4) + 2 * N


def bwd_bytes(M, N, dw_fp32):
    return M * (10 * N + 4) + 2 * N + N * (4 if dw_fp32 else 2)


def ckpt_bytes(M, N, dw_fp32):
    return 2 * fwd_bytes(M, N) + bwd_bytes(M, N, dw_fp32)


# ----------------------------------------------------------------------------- env

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(device, backend="nccl"):
    """One process per GPU; the process group's timeout bounds every collective."""
    import datetime

    import torch.distributed as dist

    kwargs = {"timeout": datetime.timedelta(seconds=120)}
    if backend == "nccl":
        kwargs["device_id"] = device
    dist.init_process_group(backend, **kwargs)
    return dist


def max_over_ranks(value, world, device):
    """The largest value over all ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(bytes_per_rank_step, steps, world, max_ms):
    """Algorithmic bytes of all ranks' steps over the slowest rank's summed step time."""
    return bytes_per_rank_step * steps * world / (max_ms * 1e-3) / 1e9


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# Host code of entry points bench.py does not call (the kernels, and the code that plans
# and launches them for bench.py, live in the other files): a change there leaves recorded
# ncu counters valid.
_DIGEST_EXCLUDED = ("host_step.cu", "noalloc.cu")


def source_digest():
    """Digest of the kernel sources and of the host code that plans and launches them."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_norm_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name in _DIGEST_EXCLUDED:
            continue
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_tag, workload):
    """DRAM bytes per launch from a committed ncu summary, if it matches the sources."""
    path = os.path.join(ROOT, "profiles", f"{kernel_tag}_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_b = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    m_s = re.search(r"source_digest:\s*([0-9a-f]+)", text)
    if not m_b or not m_s or m_s.group(1) != source_digest():
        return None
    return float(m_b.group(1))


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed loop runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(names, parts[3:7]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- oracle leg

def time_oracle(wl, min_seconds, max_rows=65536, seed=0):
    """FP64 oracle checkpointed step on a bounded row sample; returns (GB/s, rows, sec)."""
    import oracle

    rows = min(wl.M, max_rows)
    d = make_inputs(rows, wl.N, seed=seed, g_std=wl.g_std, outlier_frac=wl.outlier_frac)
    x, g, dy, w = (bf16_bits_to_f64(d[k]) for k in ("x", "g", "dy", "w"))
    done, t0 = 0, time.perf_counter()
    while True:
        oracle.ckpt_step(x, g, w, wl.eps, dy)
        done += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    gbs = ckpt_bytes(rows, wl.N, True) * done / el / 1e9
    return gbs, rows, done, el


def _oracle_worker(job):
    """One spawned process: the oracle's checkpointed step on its own seeded row sample,
    repeated until `seconds` have passed; returns (bytes done, seconds)."""
    name, rows, seed, seconds = job
    import oracle

    wl = WORKLOADS[name]
    d = make_inputs(rows, wl.N, seed=seed, g_std=wl.g_std, outlier_frac=wl.outlier_frac)
    x, g, dy, w = (bf16_bits_to_f64(d[k]) for k in ("x", "g", "dy", "w"))
    done, t0 = 0, time.perf_counter()
    while True:
        oracle.ckpt_step(x, g, w, wl.eps, dy)
        done += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            return ckpt_bytes(rows, wl.N, True) * done, el


def time_oracle_all_cores(wl, seconds, max_procs=64, rows_per_proc=8192):
    """The same oracle on every usable host core at once (one spawned process per core,
    each on its own row sample, as a row partition of the batch would run); returns
    (aggregate GB/s, processes, rows per process)."""
    import multiprocessing as mp

    procs = max(1, min(len(os.sched_getaffinity(0)), max_procs))
    rows = min(wl.M, rows_per_proc)
    jobs = [(wl.name, rows, wl.seed + 1000 + i, seconds) for i in range(procs)]
    with mp.get_context("spawn").Pool(procs) as pool:
        res = pool.map(_oracle_worker, jobs)
    gbs = sum(b / el for b, el in res) / 1e9
    return gbs, procs, rows


def run_reference(args, wl):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle  # noqa: F401

    # size the per-step row sample so the whole run stays near `ref_seconds`
    probe_rows = min(wl.M, 256)
    d = make_inputs(probe_rows, wl.N, seed=wl.seed, g_std=wl.g_std)
    px, pg, pdy, pw = (bf16_bits_to_f64(d[k]) for k in ("x", "g", "dy", "w"))
    t0 = time.perf_counter()
    oracle.ckpt_step(px, pg, pw, wl.eps, pdy)
    per_row = (time.perf_counter() - t0) / probe_rows
    budget = args.ref_seconds / max(1, args.steps + args.warmup)
    rows = int(min(wl.M, max(16, budget / max(per_row, 1e-9))))
    d = make_inputs(rows, wl.N, seed=wl.seed, g_std=wl.g_std, outlier_frac=wl.outlier_frac)
    x, g, dy, w = (bf16_bits_to_f64(d[k]) for k in ("x", "g", "dy", "w"))
    for _ in range(args.warmup):
        oracle.ckpt_step(x, g, w, wl.eps, dy)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.ckpt_step(x, g, w, wl.eps, dy)
    el = time.perf_counter() - t0
    value = ckpt_bytes(rows, wl.N, args.dw_fp32) * args.steps / el / 1e9
    sample = f"{rows} of {wl.M} rows x N={wl.N} per step (FP64 numpy oracle, one core)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "M": wl.M, "N": wl.N, "step": "ckpt (fwd, fwd, bwd)"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ----------------------------------------------------------------------------- our leg

def measure_floor(torch, dev, stream, flush, x, g, dy, y, dx, K):
    """The timing method's own floor: an empty graph (one one-element add) and torch
    elementwise kernels over the same [M, N] BF16 tensors -- y = x * g (the forward's
    reads and write) and dx = x + g * dy (three reads, one write) -- each replayed from a
    CUDA graph between the same L2 flush and events as the timed steps."""
    one = torch.zeros(1, device=dev)
    ops = {
        "empty_graph": (0, lambda: one.add_(1)),
        "torch_mul": (3 * x.numel() * 2, lambda: torch.mul(x, g, out=y)),
        "torch_addcmul": (4 * x.numel() * 2, lambda: torch.addcmul(x, g, dy, out=dx)),
    }
    reps = max(20, min(K, 200))
    out = {}
    for name, (nbytes, fn) in ops.items():
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            fn()
            fn()
        stream.wait_stream(side)
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            fn()
        for _ in range(3):
            flush.zero_()
            graph.replay()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        for a, b in evs:
            flush.zero_()
            a.record(stream)
            graph.replay()
            b.record(stream)
        torch.cuda.synchronize(dev)
        t_us = statistics.mean(a.elapsed_time(b) * 1e3 for a, b in evs)
        out[name] = {"us": t_us, "bytes": nbytes,
                     "gbs": (nbytes / (t_us * 1e-6) / 1e9) if nbytes else None}
        del graph
    return out


def run_ours(args, wl):
    import torch

    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device (the CUDA path has no CPU fallback)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist = init_dist(dev, "nccl")
    import gated_norm_b200 as gn

    M, N, eps = wl.M, wl.N, wl.eps
    det = not args.nondeterministic
    fp32 = args.dw_fp32
    d = make_inputs(M, N, seed=wl.seed + rank, g_std=wl.g_std, outlier_frac=wl.outlier_frac)

    def dev_bf16(bits):
        return torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)

    x, g, dy, w = (dev_bf16(d[k]) for k in ("x", "g", "dy", "w"))
    y, dx, dg = (torch.empty_like(x) for _ in range(3))
    rstd = torch.empty(M, dtype=torch.float32, device=dev)
    dw = torch.empty(N, dtype=torch.float32 if fp32 else torch.bfloat16, device=dev)
    ws = torch.zeros(max(gn.gnorm_bwd_workspace_bytes(M, N, det), 256), dtype=torch.uint8,
                     device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    plan_f = gn.gnorm_plan_query(0, M, N, det, sms)
    plan_b = gn.gnorm_plan_query(1, M, N, det, sms)
    fwd_kernel = ("gated_rmsnorm_fwd_direct_kernel" if plan_f["direct_loads"]
                  else "gated_rmsnorm_fwd_kernel")
    bwd_launches = 1 + (0 if plan_b["fused_reduce"] else 1)

    # The operations as the pages time them: each replayed from its own CUDA graph.
    def op_fwd():
        gn.gnorm_fwd(x, g, w, eps, y=y, rstd=rstd)

    def op_bwd():
        gn.gnorm_bwd(dy, x, g, w, rstd, dx=dx, dg=dg, dw=dw, dw_fp32=fp32, deterministic=det,
                     workspace_buf=ws)

    def op_ckpt():
        gn.gnorm_ckpt_step(x, g, w, eps, dy, y=y, rstd=rstd, dx=dx, dg=dg, dw=dw, dw_fp32=fp32,
                           deterministic=det, workspace_buf=ws)

    def capture(fn):
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            fn()
            fn()
        stream.wait_stream(side)
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            fn()
        return graph

    graphs = {"ckpt": capture(op_ckpt), "bwd": capture(op_bwd), "fwd": capture(op_fwd)}
    launches = {"ckpt": 2 + bwd_launches, "bwd": bwd_launches, "fwd": 1}
    order = ("ckpt", "bwd", "fwd")

    def one_step(evs=None):
        # one timed step: the checkpointed step (the measured unit), then the backward and
        # the forward alone for the per-operation times; L2 is flushed before each, outside
        # the events.
        for j, name in enumerate(order):
            flush.zero_()
            if evs:
                evs[2 * j].record(stream)
            graphs[name].replay()
            if evs:
                evs[2 * j + 1].record(stream)

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(K)]
    clocks = ClockSampler(local)
    if rank == 0:
        clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(K):
        one_step(evs[i])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if rank == 0 else None

    t_ckpt = [evs[i][0].elapsed_time(evs[i][1]) for i in range(K)]
    t_bwd = [evs[i][2].elapsed_time(evs[i][3]) for i in range(K)]
    t_fwd = [evs[i][4].elapsed_time(evs[i][5]) for i in range(K)]
    total_ms = max_over_ranks(float(sum(t_ckpt)), world, dev)
    step_bytes = ckpt_bytes(M, N, fp32)
    value = whole_job_gbs(step_bytes, K, world, total_ms)
    peak, peak_kind = measured_peaks()

    # one checkpointed step through the single public entry point, host buffers in and out
    e2e = None
    if args.e2e_steps > 0:
        hx, hg, hdy, hw = (t.cpu().pin_memory() for t in (x, g, dy, w))
        hy, hr, hdx, hdg, hdw = (torch.empty_like(t, device="cpu").pin_memory()
                                 for t in (y, rstd, dx, dg, dw))
        h2d = sum(t.numel() * t.element_size() for t in (hx, hg, hdy, hw))
        d2h = sum(t.numel() * t.element_size() for t in (hy, hr, hdx, hdg, hdw))
        dev_buf = torch.empty(gn.gnorm_ckpt_step_host_bytes(M, N, det), dtype=torch.uint8,
                              device=dev)

        def e2e_step():
            gn.gnorm_ckpt_step_host(hx, hg, hw, eps, hdy, y=hy, rstd=hr, dx=hdx, dg=hdg, dw=hdw,
                                    dw_fp32=fp32, deterministic=det, dev_buf=dev_buf,
                                    device=dev, stream=stream)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        e2e = {"value": whole_job_gbs(step_bytes, args.e2e_steps, world, e_ms), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e_ms / args.e2e_steps,
               "path": "gnorm_ckpt_step_host: pinned host inputs and outputs; the library "
                       "copies each step's inputs in and outputs back, chunk by chunk, "
                       "overlapping both directions of the host link with the kernels"}

    # the forward launched eagerly (no graph), same flush and events, after the timed region
    fwd_eager = []
    for i in range(min(K, 200) + 3):
        flush.zero_()
        a_ev, b_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_ev.record(stream)
        op_fwd()
        b_ev.record(stream)
        fwd_eager.append((a_ev, b_ev))
    torch.cuda.synchronize(dev)
    fwd_eager_us = statistics.mean(a_ev.elapsed_time(b_ev) for a_ev, b_ev in fwd_eager[3:]) * 1e3

    floor = measure_floor(torch, dev, stream, flush, x, g, dy, y, dx, K) if args.floor else None

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    def avg(v):
        return float(sum(v) / len(v))

    us = {"fwd": avg(t_fwd) * 1e3, "bwd": avg(t_bwd) * 1e3, "ckpt": avg(t_ckpt) * 1e3}

    def median_of_rounds(v, rounds=10):
        n = max(1, len(v) // rounds)
        meds = [statistics.median(v[i:i + n]) for i in range(0, n * (len(v) // n), n)]
        return statistics.median(meds) * 1e3

    us_median = {"fwd": median_of_rounds(t_fwd), "bwd": median_of_rounds(t_bwd),
                 "ckpt": median_of_rounds(t_ckpt)}
    gbs = {"fwd": fwd_bytes(M, N) / (us["fwd"] * 1e-6) / 1e9,
           "bwd": bwd_bytes(M, N, fp32) / (us["bwd"] * 1e-6) / 1e9,
           "ckpt": step_bytes / (us["ckpt"] * 1e-6) / 1e9}
    fwd_traffic = profiled_traffic("fwd_kernel", wl.name)
    bwd_traffic = profiled_traffic("bwd_kernel", wl.name)
    # device time of one step by kernel, from the standalone replays: the forward kernel
    # (twice) and the backward operation (kernel + second pass)
    step_us = 2 * us["fwd"] + us["bwd"]
    shares = {"fwd_kernel_x2": 2 * us["fwd"] / step_us, "bwd_op": us["bwd"] / step_us}
    cpu = cpu_all = None
    if not args.no_cpu_baseline and world == 1:  # the CPU baseline runs at N = 1 only
        c_gbs, c_rows, c_reps, c_sec = time_oracle(wl, args.cpu_seconds)
        cpu = {"value": c_gbs, "unit": "GB/s", "cores": 1, "kind": "oracle",
               "sample": f"{c_rows} of {wl.M} rows x N={N}, {c_reps} checkpointed steps "
                         f"in {c_sec:.1f} s (FP64 numpy oracle, one core)"}
        if args.cpu_all_cores:
            a_gbs, a_procs, a_rows = time_oracle_all_cores(wl, args.cpu_seconds)
            cpu_all = {"value": a_gbs, "unit": "GB/s", "cores": a_procs, "kind": "oracle",
                       "sample": f"{a_procs} processes, each {a_rows} rows x N={N} of its own, "
                                 f"checkpointed steps for {args.cpu_seconds:.0f} s "
                                 "(FP64 numpy oracle, one process per core)"}
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "M": M, "N": N, "eps": eps,
                   "step": "checkpointed step as one CUDA graph: fwd, fwd (recompute), bwd + dw reduction",
                   "deterministic": det, "dw": "fp32" if fp32 else "bf16",
                   "l2": "flushed between steps (256 MiB write, outside the timed events)",
                   "parallelism": f"dp{world} (independent rows per rank, no collective)"},
        "us_per_call": us,
        "us_median_of_round_medians": us_median,
        "us_fwd_eager": fwd_eager_us,
        "timing": "fwd, bwd, ckpt each replayed from its own CUDA graph (fwdg, bwdg, ckptg)",
        "gbs": gbs,
        "frac_of_peak": {k: v / peak for k, v in gbs.items()},
        "roofline": {"bound": "hbm",
                     "kernel": f"{fwd_kernel} (one launch per fwdg replay)",
                     "achieved": gbs["fwd"], "peak": peak, "peak_kind": peak_kind,
                     "unit": "GB/s", "frac": gbs["fwd"] / peak,
                     "algorithmic_bytes_per_launch": fwd_bytes(M, N),
                     "traffic": fwd_traffic},
        "roofline_bwd": {"bound": "hbm",
                         "kernel": "gnorm_bwd (backward kernel + dw second pass, one bwdg "
                                   "replay)",
                         "achieved": gbs["bwd"], "peak": peak, "peak_kind": peak_kind,
                         "unit": "GB/s", "frac": gbs["bwd"] / peak,
                         "algorithmic_bytes_per_launch": bwd_bytes(M, N, fp32),
                         "traffic": bwd_traffic},
        "step_shares": shares,
        "cpu_baseline": cpu,
        "cpu_baseline_all_cores": cpu_all,
        "e2e": e2e,
        "gpu_launches": sum(launches.values()) * K,
        "clocks": clk,
    }
    if floor is not None:
        line["floor"] = floor
    print(json.dumps(line))
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--nondeterministic", action="store_true")
    ap.add_argument("--dw-fp32", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-cpu-all-cores", dest="cpu_all_cores", action="store_false",
                    help="skip the oracle timed on all host cores")
    ap.add_argument("--floor", action="store_true",
                    help="also time an empty graph and torch elementwise kernels the same way")
    ap.add_argument("--ref-seconds", type=float, default=60.0,
                    help="target duration of the reference (oracle) arm")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    wl = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_ours(args, wl)


if __name__ == "__main__":
    sys.exit(main())
