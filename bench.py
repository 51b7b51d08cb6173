"""Benchmark of the SiLU-gated RMSNorm training step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--nondeterministic] [--dw-bf16] [--flush]

A step is one checkpointed training step over one batch of seeded synthetic rows:
forward, then the recompute forward and the backward (one kernel where the backward stages
its rows) with the dw reduction -- every stage of the path -- replayed from one CUDA graph
("ckptg").  The default workload is 262144 x 256 with
an FP32 dw, deterministic (the checkpointed step with FP32 dw, "stepg_f32" in the pages'
list of operations).  The timed region is K steps.  When the inputs are larger than L2
(x and g alone exceed it at every large workload) the K replays run back to back between
one pair of CUDA events; otherwise L2 is flushed before every replay, outside a pair of
events around that replay.  Before the timed region the forward ("fwdg"), the backward
("bwdg") and the fused forward + backward are timed the same way from their own graphs, for
the per-operation times and the roofline of each; after it the operations are also timed
with a cold L2 before every replay (`us_per_call_cold_l2`), called eagerly through the
Python binding without a graph (`us_per_call_eager`, the pages' "fwd" column), and
`per_config` gives them for the other large workloads.  `value` is the checkpointed step's algorithmic HBM bytes of the whole job / the
max-over-ranks time of the K steps (GB/s).

Under torchrun (N > 1) every rank runs its own batch (weak scaling, no collective on the
data path; the rows of a data-parallel batch are independent).  `--impl reference` times
the FP64 CPU oracle on a bounded sample of the same workload (rank 0 only).  `--floor`
adds the same measurement of an empty graph and of torch elementwise kernels that move the
forward's and backward's main streams.
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
DEFAULT_WORKLOAD = "mid_262144x256"
PER_CONFIG_WORKLOADS = ("long_368640x128", "wide_16384x4096", "mid_262144x256")
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20
OP_REPS = 100  # replays per loop when an operation is timed alone


# ----------------------------------------------------------------------------- bytes

def fwd_bytes(M, N):
    return M * (6 * N + 4) + 2 * N


def bwd_bytes(M, N, dw_fp32):
    return M * (10 * N + 4) + 2 * N + N * (4 if dw_fp32 else 2)


def ckpt_bytes(M, N, dw_fp32):
    return 2 * fwd_bytes(M, N) + bwd_bytes(M, N, dw_fp32)


def fwd_bwd_bytes(M, N, dw_fp32):
    """The fused forward + backward of the same rows: read x, g, dy; write y, rstd, dx, dg
    (12N + 4 per row), w once and dw."""
    return M * (12 * N + 4) + 2 * N + N * (4 if dw_fp32 else 2)


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


def _code_only(text):
    """C/C++/CUDA source without its comments and blank lines (the sources hold no string
    literal with a comment marker), so that a comment edit keeps the digest."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def source_digest(csrc=None):
    """Digest of the kernel sources and of the host code that plans and launches them
    (their code, not their comments)."""
    h = hashlib.sha256()
    csrc = csrc or os.path.join(ROOT, "gated_norm_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name in _DIGEST_EXCLUDED:
            continue
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + _code_only(f.read()).encode())
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
    value = ckpt_bytes(rows, wl.N, not args.dw_bf16) * args.steps / el / 1e9
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

def l2_bytes(torch, dev):
    try:
        return int(torch.cuda.get_device_properties(dev).L2_cache_size)
    except Exception:
        return 126 * 1000 * 1000


def capture_graph(torch, dev, stream, fn, launches=1):
    """A CUDA graph holding `launches` consecutive calls of `fn` (captured on a side stream
    after two eager calls, which also set up any per-device state)."""
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        fn()
        fn()
    stream.wait_stream(side)
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        for _ in range(launches):
            fn()
    return graph


class _Eager:
    """A callable with a graph's replay() interface, for Timer."""

    def __init__(self, fn):
        self.replay = fn


class Timer:
    """CUDA-event timing of graph replays on `stream`.

    streamed=True: the replays run back to back between one pair of events (the inputs of
    every operation are larger than L2, so one replay finds nothing of the previous one's
    rows in L2); the per-replay time is the total over the count.
    streamed=False: L2 is flushed (a write of `flush`, larger than L2) before every replay,
    outside a pair of events around that replay."""

    def __init__(self, torch, stream, flush, streamed):
        self.torch, self.stream, self.flush, self.streamed = torch, stream, flush, streamed

    def run(self, graph, reps):
        """Total device milliseconds of `reps` replays, and the per-replay list (for the
        streamed mode, each replay's own events sit inside the outer pair)."""
        torch, s = self.torch, self.stream
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(reps)]
        if self.streamed:
            a0, b0 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(s)
            for _ in range(reps):
                graph.replay()
            b0.record(s)
            torch.cuda.synchronize()
            return a0.elapsed_time(b0), None
        for a, b in ev:
            self.flush.zero_()
            a.record(s)
            graph.replay()
            b.record(s)
        torch.cuda.synchronize()
        per = [a.elapsed_time(b) for a, b in ev]
        return float(sum(per)), per

    def cold(self, graph, reps):
        """Mean ms of `reps` replays each after an L2 flush (events around each replay)."""
        saved = self.streamed
        self.streamed = False
        try:
            total, _ = self.run(graph, reps)
        finally:
            self.streamed = saved
        return total / reps


def measure_floor(torch, dev, stream, timer, x, g, dy, y, dx, reps):
    """The timing method's own floor: an empty graph (one one-element add) and torch
    elementwise kernels over the same [M, N] BF16 tensors -- y = x * g (the forward's
    reads and write) and dx = x + g * dy (three reads, one write) -- timed exactly as the
    operations are."""
    one = torch.zeros(1, device=dev)
    ops = {
        "empty_graph": (0, lambda: one.add_(1)),
        "torch_mul": (3 * x.numel() * 2, lambda: torch.mul(x, g, out=y)),
        "torch_addcmul": (4 * x.numel() * 2, lambda: torch.addcmul(x, g, dy, out=dx)),
    }
    out = {}
    for name, (nbytes, fn) in ops.items():
        graph = capture_graph(torch, dev, stream, fn)
        timer.run(graph, 3)
        total, _ = timer.run(graph, reps)
        t_us = total / reps * 1e3
        out[name] = {"us": t_us, "bytes": nbytes,
                     "gbs": (nbytes / (t_us * 1e-6) / 1e9) if nbytes else None}
        del graph
    return out


class Problem:
    """Device tensors of one workload and CUDA graphs of its three operations (fwdg, bwdg,
    ckptg, as the pages name them)."""

    def __init__(self, torch, gn, dev, stream, wl, det, fp32, seed_offset=0, graphs=True,
                 knobs=None):
        knobs = knobs or {}
        self.torch, self.gn, self.wl = torch, gn, wl
        self.M, self.N, self.eps = wl.M, wl.N, wl.eps
        self.det, self.fp32 = det, fp32
        d = make_inputs(wl.M, wl.N, seed=wl.seed + seed_offset, g_std=wl.g_std,
                        outlier_frac=wl.outlier_frac, outlier_scale=wl.outlier_scale)

        def dev_bf16(bits):
            return torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)

        self.x, self.g, self.dy, self.w = (dev_bf16(d[k]) for k in ("x", "g", "dy", "w"))
        self.y, self.dx, self.dg = (torch.empty_like(self.x) for _ in range(3))
        self.rstd = torch.empty(wl.M, dtype=torch.float32, device=dev)
        self.dw = torch.empty(wl.N, dtype=torch.float32 if fp32 else torch.bfloat16, device=dev)
        self.ws = torch.zeros(max(gn.gnorm_bwd_workspace_bytes(wl.M, wl.N, det), 256),
                              dtype=torch.uint8, device=dev)
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        self.plan_f = gn.gnorm_plan_query(0, wl.M, wl.N, det, sms)
        self.plan_b = gn.gnorm_plan_query(1, wl.M, wl.N, det, sms)
        self.bwd_launches = 1 + (0 if self.plan_b["fused_reduce"] else 1)
        # the recompute forward and the backward run as one kernel where the backward's
        # plan stages its rows (and the fuse_fwd_bwd knob does not say otherwise)
        self.fused = (not self.plan_b["direct_loads"]) and knobs.get("fuse_fwd_bwd", 0) != 2
        fb = self.bwd_launches + (0 if self.fused else 1)
        self.launches = {"ckpt": 1 + fb, "fwd_bwd": fb, "bwd": self.bwd_launches, "fwd": 1}
        self.graphs = {name: capture_graph(torch, dev, stream, fn)
                       for name, fn in (("ckpt", self.op_ckpt), ("fwd_bwd", self.op_fwd_bwd),
                                        ("bwd", self.op_bwd), ("fwd", self.op_fwd))
                       } if graphs else {}

    def op_fwd(self):
        self.gn.gnorm_fwd(self.x, self.g, self.w, self.eps, y=self.y, rstd=self.rstd)

    def op_bwd(self):
        self.gn.gnorm_bwd(self.dy, self.x, self.g, self.w, self.rstd, dx=self.dx, dg=self.dg,
                          dw=self.dw, dw_fp32=self.fp32, deterministic=self.det,
                          workspace_buf=self.ws)

    def op_fwd_bwd(self):
        self.gn.gnorm_fwd_bwd(self.x, self.g, self.w, self.eps, self.dy, y=self.y,
                              rstd=self.rstd, dx=self.dx, dg=self.dg, dw=self.dw,
                              dw_fp32=self.fp32, deterministic=self.det, workspace_buf=self.ws)

    def op_ckpt(self):
        self.gn.gnorm_ckpt_step(self.x, self.g, self.w, self.eps, self.dy, y=self.y,
                                rstd=self.rstd, dx=self.dx, dg=self.dg, dw=self.dw,
                                dw_fp32=self.fp32, deterministic=self.det, workspace_buf=self.ws)

    def fwd_kernel(self):
        return ("gated_rmsnorm_fwd_direct_kernel" if self.plan_f["direct_loads"]
                else "gated_rmsnorm_fwd_kernel")

    def bytes(self):
        return {"fwd": fwd_bytes(self.M, self.N), "bwd": bwd_bytes(self.M, self.N, self.fp32),
                "fwd_bwd": fwd_bwd_bytes(self.M, self.N, self.fp32),
                "ckpt": ckpt_bytes(self.M, self.N, self.fp32)}

    def step_dram_bytes(self):
        """Bytes the checkpointed step must move as this library runs it: the forward, then
        the fused forward + backward (or the forward and the backward apart)."""
        b = self.bytes()
        return b["fwd"] + (b["fwd_bwd"] if self.fused else b["fwd"] + b["bwd"])

    def release(self):
        self.graphs.clear()


def op_times(timer, prob, reps):
    """Mean device microseconds per replay of fwdg, bwdg, the fused forward + backward and
    ckptg."""
    out = {}
    for name in ("fwd", "bwd", "fwd_bwd", "ckpt"):
        timer.run(prob.graphs[name], 3)
        total, _ = timer.run(prob.graphs[name], reps)
        out[name] = total / reps * 1e3
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

    knobs = parse_tune(args.tune)
    if knobs:
        gn.gnorm_set_tuning(**knobs)
    det = not args.nondeterministic
    fp32 = not args.dw_bf16
    stream = torch.cuda.current_stream(dev)
    l2 = l2_bytes(torch, dev)
    flush = torch.empty(max(L2_FLUSH_BYTES, 2 * l2), dtype=torch.uint8, device=dev)
    prob = Problem(torch, gn, dev, stream, wl, det, fp32, seed_offset=rank, knobs=knobs)
    M, N = prob.M, prob.N
    # The smallest operation's inputs: the forward reads x and g.
    streamed = (not args.flush) and 2 * M * N * 2 > l2
    timer = Timer(torch, stream, flush, streamed)
    ckpt_graph = prob.graphs["ckpt"]

    for _ in range(args.warmup):
        if not streamed:
            flush.zero_()
        ckpt_graph.replay()
    torch.cuda.synchronize()

    K = args.steps
    # each operation alone, timed the same way from its own graph in loops of at most
    # OP_REPS replays, before the sustained timed region: a kernel timed alone, like the
    # measured copy bandwidth it is compared with (after a long loop of steps the board's
    # power cap slows the fused forward + backward by up to 3%)
    us = op_times(timer, prob, min(K, OP_REPS))
    clocks = ClockSampler(local)
    if rank == 0:
        clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    total_ms, per_step = timer.run(ckpt_graph, K)   # the timed region: K checkpointed steps
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    total_ms = max_over_ranks(total_ms, world, dev)
    step_bytes = ckpt_bytes(M, N, fp32)
    value = whole_job_gbs(step_bytes, K, world, total_ms)
    peak, peak_kind = measured_peaks()

    us["ckpt"] = total_ms / K * 1e3
    # the same operations with a cold L2 before every replay, events around each replay
    # (this also counts each replay's own launch latency)
    cold_reps = max(10, min(K, 100))
    us_cold = {name: prob_t * 1e3 for name, prob_t in
               ((n, timer.cold(prob.graphs[n], cold_reps))
                for n in ("fwd", "bwd", "fwd_bwd", "ckpt"))}
    # the same operations called eagerly (no graph): each call goes through the binding and
    # the C entry point, which plan and launch on the stream
    eager_reps = max(10, min(K, OP_REPS))
    us_eager = {}
    for name, fn in (("fwd", prob.op_fwd), ("bwd", prob.op_bwd), ("fwd_bwd", prob.op_fwd_bwd),
                     ("ckpt", prob.op_ckpt)):
        call = _Eager(fn)
        timer.run(call, 3)
        us_eager[name] = timer.run(call, eager_reps)[0] / eager_reps * 1e3
    per_config = {}
    if args.per_config and world == 1:
        for name in PER_CONFIG_WORKLOADS:
            if name == wl.name:
                continue
            other = Problem(torch, gn, dev, stream, WORKLOADS[name], det, fp32, knobs=knobs)
            o_streamed = (not args.flush) and 2 * other.M * other.N * 2 > l2
            o_timer = Timer(torch, stream, flush, o_streamed)
            t = op_times(o_timer, other, args.per_config_steps)
            b = other.bytes()
            per_config[name] = {
                "M": other.M, "N": other.N, "us": t,
                "gbs": {k: b[k] / (t[k] * 1e-6) / 1e9 for k in t},
                "frac_of_peak": {k: b[k] / (t[k] * 1e-6) / 1e9 / peak for k in t if k != "ckpt"},
                "frac_of_peak_ckpt_dram": other.step_dram_bytes() / (t["ckpt"] * 1e-6) / 1e9
                                          / peak,
                "fwd_kernel": other.fwd_kernel(),
                "l2": "inputs larger than L2, replays back to back" if o_streamed
                      else "L2 flushed before every replay",
            }
            other.release()
            del other
            torch.cuda.synchronize()
    clk = clocks.stop() if rank == 0 else None

    # one checkpointed step through the public host-buffer entry point: inputs copied in
    # and outputs copied back every step
    e2e = None
    if args.e2e_steps > 0:
        hx, hg, hdy, hw = (t.cpu().pin_memory() for t in (prob.x, prob.g, prob.dy, prob.w))
        hy, hr, hdx, hdg, hdw = (torch.empty_like(t, device="cpu").pin_memory()
                                 for t in (prob.y, prob.rstd, prob.dx, prob.dg, prob.dw))
        h2d = sum(t.numel() * t.element_size() for t in (hx, hg, hdy, hw))
        d2h = sum(t.numel() * t.element_size() for t in (hy, hr, hdx, hdg, hdw))
        dev_buf = torch.empty(gn.gnorm_ckpt_step_host_bytes(M, N, det), dtype=torch.uint8,
                              device=dev)

        def e2e_step():
            gn.gnorm_ckpt_step_host(hx, hg, hw, prob.eps, hdy, y=hy, rstd=hr, dx=hdx, dg=hdg,
                                    dw=hdw, dw_fp32=fp32, deterministic=det, dev_buf=dev_buf,
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
        del dev_buf

    floor = (measure_floor(torch, dev, stream, timer, prob.x, prob.g, prob.dy, prob.y, prob.dx,
                           max(20, min(K, 200))) if args.floor else None)

    if world > 1:
        dist.barrier()
        prob.release()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    b = prob.bytes()
    gbs = {k: b[k] / (us[k] * 1e-6) / 1e9 for k in us}
    gbs_cold = {k: b[k] / (us_cold[k] * 1e-6) / 1e9 for k in us_cold}
    traffic = {k: profiled_traffic(f"{k}_kernel", wl.name) for k in ("fwd", "bwd", "fwd_bwd")}
    # device time of one step by operation, from the standalone replays: the forward kernel,
    # then the fused forward + backward (kernel + dw pass), or, unfused, the forward twice
    # and the backward (kernel + dw pass)
    if prob.fused:
        step_us = us["fwd"] + us["fwd_bwd"]
        shares = {"fwd_kernel": us["fwd"] / step_us, "fwd_bwd_op": us["fwd_bwd"] / step_us}
    else:
        step_us = 2 * us["fwd"] + us["bwd"]
        shares = {"fwd_kernel_x2": 2 * us["fwd"] / step_us, "bwd_op": us["bwd"] / step_us}
    fwd_name = f"{prob.fwd_kernel()} (one launch per fwdg replay)"
    objs = {
        "fwd": fwd_name,
        "bwd": "gnorm_bwd (backward kernel + dw second pass, one bwdg replay)",
        "fwd_bwd": ("gnorm_fwd_bwd (the forward fused into the backward kernel, + dw second "
                    "pass; one replay)" if prob.fused else
                    "gnorm_fwd_bwd (forward kernel, backward kernel, dw pass; one replay)"),
    }

    def roofline_of(key):
        return {"bound": "hbm", "kernel": objs[key], "achieved": gbs[key], "peak": peak,
                "peak_kind": peak_kind, "unit": "GB/s", "frac": gbs[key] / peak,
                "algorithmic_bytes_per_launch": b[key], "traffic": traffic[key]}

    # the operation with the largest share of the step's device time
    dominant = "fwd_bwd" if (prob.fused and us["fwd_bwd"] > us["fwd"]) else "fwd"
    dram_step = prob.step_dram_bytes()
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
    l2_note = (f"inputs larger than L2 ({2 * M * N * 2 / 1e6:.0f} MB of x and g per forward "
               f"against {l2 / 1e6:.0f} MB of L2): replays back to back, no flush"
               if streamed else
               f"L2 flushed before every replay ({flush.numel() >> 20} MiB write, outside "
               "the timed events)")
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "M": M, "N": N, "eps": prob.eps,
                   "step": "checkpointed step as one CUDA graph: fwd, then the recompute "
                           "fwd and the bwd (fused into one kernel where the backward stages "
                           "its rows), + dw reduction",
                   "deterministic": det, "dw": "fp32" if fp32 else "bf16",
                   "l2": l2_note,
                   "parallelism": f"dp{world} (independent rows per rank, no collective)",
                   **({"tuning": knobs} if knobs else {})},
        "us_per_call": us,
        "timing": ("ckptg replayed K times back to back between two CUDA events (the timed "
                   "region); before it, fwdg, bwdg and the fused forward + backward timed the "
                   "same way from their own graphs, at most 100 replays each"
                   if streamed else
                   "each of ckptg, fwdg, bwdg replayed from its own CUDA graph between two "
                   "CUDA events after an L2 flush"),
        "gbs": gbs,
        # each operation's algorithmic bytes over its time, against the HBM peak; for the
        # step the bytes are the counted 2 x forward + backward (see step_bytes_note), so its
        # fraction of the HBM peak is the DRAM one below
        "frac_of_peak": {k: v / peak for k, v in gbs.items() if k != "ckpt"},
        "frac_of_peak_ckpt_dram": (dram_step / (us["ckpt"] * 1e-6) / 1e9) / peak,
        "us_per_call_cold_l2": us_cold,
        "frac_of_peak_cold_l2": {k: v / peak for k, v in gbs_cold.items() if k != "ckpt"},
        "cold_l2_note": (f"{cold_reps} replays each after a {flush.numel() >> 20} MiB L2 flush, "
                         "events around each replay, so each also counts its graph's launch "
                         "latency"),
        "us_per_call_eager": us_eager,
        "eager_note": (f"{eager_reps} calls of each operation through the Python binding "
                       "without a graph, timed like the graph replays (back to back, or each "
                       "after an L2 flush); each call's host path is in the time where it is "
                       "longer than the kernels"),
        "roofline": roofline_of(dominant),
        "roofline_fwd": roofline_of("fwd"),
        "roofline_bwd": roofline_of("bwd"),
        "roofline_fwd_bwd": roofline_of("fwd_bwd"),
        "dram_bytes_per_step": dram_step,
        "dram_gbs": dram_step * K * world / (total_ms * 1e-3) / 1e9,
        "step_bytes_note": ("value counts the step as 2 x forward + backward (the pages' "
                            "ckptg); the recompute forward runs inside the backward kernel, "
                            "which reads x and g once for both, so the step moves "
                            "dram_bytes_per_step to DRAM; dram_gbs is that over the same time"
                            if prob.fused else
                            "the step runs as three kernels: dram_bytes_per_step equals the "
                            "counted bytes"),
        "step_shares": shares,
        "per_config": per_config or None,
        "cpu_baseline": cpu,
        "cpu_baseline_all_cores": cpu_all,
        "e2e": e2e,
        "gpu_launches": prob.launches["ckpt"] * K,
        "clocks": clk,
    }
    if floor is not None:
        line["floor"] = floor
    print(json.dumps(line))
    return 0


def parse_tune(items):
    """--tune KNOB=VALUE pairs -> a dict of gnorm_tuning fields."""
    out = {}
    for it in items:
        k, _, v = it.partition("=")
        if not k or not v:
            raise SystemExit(f"bench.py: --tune wants KNOB=VALUE, got {it!r}")
        out[k.strip()] = int(v)
    return out


def run_profile(args, wl):
    """Only `--profile-op` on the workload's inputs: one untimed call, then `--reps` calls,
    nothing else on the GPU (a short, fixed launch list for ncu captures)."""
    import torch

    import gated_norm_b200 as gn

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    knobs = parse_tune(args.tune)
    if knobs:
        gn.gnorm_set_tuning(**knobs)
    prob = Problem(torch, gn, dev, torch.cuda.current_stream(dev), wl,
                   not args.nondeterministic, not args.dw_bf16, graphs=False, knobs=knobs)
    fn = {"fwd": prob.op_fwd, "bwd": prob.op_bwd, "fwd_bwd": prob.op_fwd_bwd,
          "ckpt": prob.op_ckpt}[args.profile_op]
    torch.cuda.synchronize()
    for _ in range(args.reps):
        fn()
    torch.cuda.synchronize()
    err = gn.gnorm_device_error(reset=True)
    prob.release()
    print(json.dumps({"profile_op": args.profile_op, "workload": wl.name, "reps": args.reps,
                      "tune": knobs, "plan_fwd": prob.plan_f, "plan_bwd": prob.plan_b,
                      "device_error": err}))
    return 0 if err == 0 else 1


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--nondeterministic", action="store_true")
    ap.add_argument("--dw-bf16", action="store_true", help="BF16 dw (default: FP32 dw)")
    ap.add_argument("--flush", action="store_true",
                    help="flush L2 before every replay even when the inputs exceed L2")
    ap.add_argument("--no-per-config", dest="per_config", action="store_false",
                    help="skip the per-operation times of the other large workloads")
    ap.add_argument("--per-config-steps", type=int, default=50)
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-cpu-all-cores", dest="cpu_all_cores", action="store_false",
                    help="skip the oracle timed on all host cores")
    ap.add_argument("--floor", action="store_true",
                    help="also time an empty graph and torch elementwise kernels the same way")
    ap.add_argument("--ref-seconds", type=float, default=60.0,
                    help="target duration of the reference (oracle) arm")
    ap.add_argument("--tune", action="append", default=[], metavar="KNOB=VALUE",
                    help="a gnorm_tuning knob for this run (repeatable; recorded in config)")
    ap.add_argument("--profile-op", choices=("fwd", "bwd", "fwd_bwd", "ckpt"),
                    help="run only this operation --reps times and exit (for ncu captures)")
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--rows", type=int, default=0,
                    help="override the workload's row count (same distributions; for "
                         "smaller profiling cases)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    wl = WORKLOADS[args.workload]
    if args.rows:
        wl = wl.scaled(args.rows)
    if args.profile_op:
        return run_profile(args, wl)
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_ours(args, wl)


if __name__ == "__main__":
    sys.exit(main())
