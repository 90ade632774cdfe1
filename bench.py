"""Benchmark of the SA compression step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step is one SA layer over the whole batch: the fused tensor-core pass
over X plus the finalize pass, through the C ABI (libsa.so).  The default
workload is 16 users x 100K behaviours, d = 128, k = 128, bf16 (X drawn from
a 512-component Gaussian mixture) -- the configuration whose roofline is the
target.  X is 409.6 MB, larger than the 126 MB L2, so every step streams it
from HBM.

Prints one JSON line (rank 0).  ``value`` is rows/s over all ranks with X
resident in HBM; ``e2e`` is the same metric through the host-buffer entry
point, host->device copy of X and device->host copy of the sketches inside
the timed region; ``roofline`` is the fused kernel against the measured HBM
peak; ``cpu_baseline`` is the CPU oracle timed on a bounded sample.

With --gpus N > 1 (launched by torchrun) every rank runs its own batch
(users are independent; no collective on the data path) and the timing is
the max over ranks (weak scaling).  ``--impl reference`` times the CPU
oracle instead (rank 0 only).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
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

from synthetic import WORKLOADS, generate, user_queries  # noqa: E402

METRIC = "SA history rows/sec and % of roofline (max(HBM, bf16 TC)) on 1 B200"
DEFAULT_WORKLOAD = "batch16_n100k_d128_k128_mixture_bf16"
L2_BYTES = 126e6
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
KERNEL_SOURCES = ["sketch_attention_compression_b200/csrc/sa_fused.cu",
                  "sketch_attention_compression_b200/csrc/sa_plan.h",
                  "sketch_attention_compression_b200/csrc/sa_ptx.cuh",
                  "sketch_attention_compression_b200/csrc/sa_internal.h"]
# ncu summaries that carry the DRAM traffic of the dominant kernel, per workload
TRAFFIC_FILES = {
    DEFAULT_WORKLOAD: os.path.join(ROOT, "profiles", "fused_sa_batch16_n100k_d128_k128.md"),
    "batch16_n100k_d128_k1000_mixture_bf16":
        os.path.join(ROOT, "profiles", "fused_sa_cluster_batch16_n100k_d128_k1000.md"),
}


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def load_traffic(workload: str):
    """DRAM bytes per launch of the fused kernel on `workload` from the
    committed ncu summary, if there is one and it was taken on the current
    kernel source (else None)."""
    path = TRAFFIC_FILES.get(workload)
    if path is None or not os.path.exists(path):
        return None
    text = open(path).read()
    m_hash = re.search(r"kernel_source_hash:\s*([0-9a-f]+)", text)
    m_tr = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_hash or not m_tr or m_hash.group(1) != kernel_source_hash():
        return None
    return float(m_tr.group(1))


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    """Samples the SM clock, power draw and clock-event (throttle) reasons of
    one GPU while the timed region runs.  Reads only; changes no setting.

    NVML is polled about every millisecond from a thread, so that even a
    timed region of a few milliseconds gets samples; without NVML it falls
    back to nvidia-smi at 50 ms."""

    REASONS = [("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap")]

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.samples = []  # (sm_mhz, max_mhz, watts, reason_bits)
        self.stop_flag = threading.Event()
        self.thread = None
        self.nvml = None
        self.proc = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            handle = pynvml.nvmlDeviceGetHandleByUUID(self.uuid)
            self.nvml = (pynvml, handle)
            self.thread = threading.Thread(target=self._poll_nvml, daemon=True)
        except Exception:
            self.nvml = None
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "--query-gpu=uuid,clocks.sm,clocks.max.sm,power.draw,"
                     "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                     "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                     "--format=csv,noheader,nounits", "-lms", "50"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except OSError:
                return
            self.thread = threading.Thread(target=self._read_smi, daemon=True)
        self.thread.start()

    def _poll_nvml(self):
        pynvml, h = self.nvml
        bits = {name: getattr(pynvml, const, 0) for name, const in self.REASONS}
        mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        while not self.stop_flag.is_set():
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0
                rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((sm, mx, pw, {n for n, b in bits.items() if rs & b}))
            except Exception:
                pass
            time.sleep(0.001)

    def _read_smi(self):
        names = [n for n, _ in self.REASONS]
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8 or (self.uuid and parts[0] != self.uuid):
                continue
            try:
                self.samples.append((float(parts[1]), float(parts[2]), float(parts[3]),
                                     {n for n, v in zip(names, parts[4:8]) if v.lower() == "active"}))
            except ValueError:
                continue

    def mark(self) -> int:
        return len(self.samples)

    def stop(self):
        self.stop_flag.set()
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, first: int = 0, last=None):
        rows = self.samples[first:last]
        if not rows:
            return None
        reasons = set()
        for r in rows:
            reasons |= r[3]
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows),
                "power_w_median": round(statistics.median(r[2] for r in rows), 1),
                "reasons": sorted(reasons), "samples": len(rows),
                "source": "nvml" if self.nvml else "nvidia-smi"}


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline / reference arm)
# ---------------------------------------------------------------------------

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        if info:
            return int(max(i.get("num_threads", 1) for i in info))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_rows_per_s(inp: dict, budget_s: float, users=None, queries=None):
    """Runs the oracle user by user until `budget_s` has elapsed (at least one
    user); returns (rows/s, rows, seconds, users).  With `queries` (B, k, d),
    user b is queried by queries[b] in place of P."""
    from oracle import sa_user
    offs = inp["offsets"]
    order = list(range(len(offs) - 1)) if users is None else users
    rows = 0
    done = []
    t0 = time.perf_counter()
    for b in order:
        lo, hi = int(offs[b]), int(offs[b + 1])
        sa_user(inp["X"][lo:hi], inp["P"] if queries is None else queries[b], inp["W_Q"],
                inp["W_K"], inp["scale"])
        rows += hi - lo
        done.append(b)
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return rows / dt, rows, dt, done


def workload_inputs(args, seed=None) -> dict:
    """The named workload; with --users U, only its first U users (a smaller
    case of the same shapes, e.g. for a profiler capture)."""
    inp = generate(args.workload, seed=seed)
    if args.users and args.users < len(inp["offsets"]) - 1:
        offs = inp["offsets"][: args.users + 1].copy()
        inp["offsets"] = offs
        inp["X"] = inp["X"][: int(offs[-1])]
    return inp


class RankGroup:
    """The ranks of one bench run: one process per GPU, with
    torch.distributed only for the barrier around each timed region and the
    reductions of the timings and row counts (the path itself has no
    collective).  The reduction tensors live on `device`: the rank's GPU
    with NCCL, the CPU with gloo."""

    def __init__(self, world: int, device):
        self.world = world
        self.device = device

    def barrier(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()

    def _reduce(self, x: float, op: str) -> float:
        if self.world == 1:
            return float(x)
        import torch
        import torch.distributed as dist
        t = torch.tensor([float(x)], dtype=torch.float64, device=self.device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
        return float(t.item())

    def max(self, x: float) -> float:
        return self._reduce(x, "max")

    def sum(self, x: float) -> float:
        return self._reduce(x, "sum")


def init_rank_group(world: int, local_rank: int, backend: str = "nccl") -> RankGroup:
    """Joins the process group of a torchrun launch (env:// rendezvous) and
    returns the bench's view of it; a single process needs no group."""
    import torch
    if world == 1:
        return RankGroup(1, torch.device("cuda", local_rank) if backend == "nccl" else "cpu")
    import datetime

    import torch.distributed as dist
    if backend == "nccl":
        torch.cuda.set_device(local_rank)
        device = torch.device("cuda", local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    else:
        device = torch.device("cpu")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return RankGroup(world, device)


def rank_seed(workload: str, rank: int) -> int:
    """Each rank draws its own batch of the workload (weak scaling)."""
    return WORKLOADS[workload].seed + rank


def run_reference(args, rank: int):
    if rank != 0:
        return
    inp = workload_inputs(args)
    w = WORKLOADS[args.workload]
    offs = inp["offsets"]
    # one step = the oracle over one user's history (a bounded sample)
    user = 0
    step_rows = int(offs[user + 1] - offs[user])
    for _ in range(args.warmup):
        oracle_rows_per_s(inp, 0.0, users=[user])
    times = []
    for _ in range(args.steps):
        _, rows, dt, _ = oracle_rows_per_s(inp, 0.0, users=[user])
        times.append(dt)
    total = sum(times)
    value = step_rows * args.steps / total
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "rows/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "users": len(offs) - 1, "d": w.d, "k": w.k,
                   "step_sample": f"user {user} ({step_rows} rows) per step"},
        "cpu_baseline": {"value": value, "unit": "rows/s", "cores": cores, "kind": "oracle",
                         "sample": f"user {user} of the workload, {step_rows} rows per step"},
        "e2e": {"value": value, "unit": "rows/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args, rank: int, world: int, local_rank: int, ranks: RankGroup):
    import torch

    from sketch_attention_compression_b200 import SketchQuery, load_library, read_device_status

    load_library()  # fails loudly if the CUDA library is missing
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = WORKLOADS[args.workload]
    inp = workload_inputs(args, seed=rank_seed(args.workload, rank))
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    X = torch.from_numpy(inp["X"]).to(dev).to(tdt)
    P, W_Q, W_K = (torch.from_numpy(inp[k]).to(dev).to(tdt) for k in ("P", "W_Q", "W_K"))
    offsets = torch.from_numpy(inp["offsets"]).to(dev)
    B = len(inp["offsets"]) - 1
    N = int(inp["offsets"][-1])
    elem = 2 if w.dtype == "bf16" else 4
    # An X that fits in L2 would let timed iterations hit in L2: the timed
    # loops then rotate over enough copies that each iteration's X was
    # evicted since its last use (copies x size > 2 x L2).
    x_bytes = float(N) * w.d * elem
    n_copies = 1 if x_bytes > L2_BYTES else int(math.ceil(2 * L2_BYTES / max(x_bytes, 1.0)))
    Xs = [X] + [X.clone() for _ in range(n_copies - 1)]

    stream = torch.cuda.current_stream(dev)
    q = SketchQuery(P, W_Q, W_K, inp["scale"], stream=stream)
    Xt = torch.empty((B, w.k, w.d), dtype=torch.float32, device=dev)
    m = torch.empty((B, w.k), dtype=torch.float32, device=dev)
    uq = args.user_queries
    if uq:
        # The SA step of a refinement layer: every user queried by its own
        # k x d matrix (seeded like P), the same X and weights.
        Q_host = torch.from_numpy(user_queries(B, w.k, w.d, seed=rank_seed(args.workload, rank)
                                               + 100)).pin_memory()
        Qd = Q_host.to(dev)
        ws = torch.empty(q.workspace_bytes_user_queries(B, N), dtype=torch.uint8, device=dev)

        def step(x):
            q.forward_user_queries(Qd, x, offsets, Xt, m, ws, stream=stream)

        def first_pass(x):
            q.partials_user_queries(Qd, x, offsets, Xt, m, ws, stream=stream)
    else:
        ws = q.new_workspace(B, N)

        def step(x):
            q.forward(x, offsets, Xt, m, ws, stream=stream)

        def first_pass(x):
            q.partials(x, offsets, Xt, m, ws, stream=stream)
    kernels_per_step = 3 if uq else 2

    barrier = ranks.barrier
    max_over_ranks = ranks.max

    # warm-up (also checks the device flags once)
    for i in range(max(args.warmup, 1)):
        step(Xs[i % n_copies])
    if read_device_status(ws, stream) != 0:
        raise RuntimeError("device flags raised during warm-up")

    clocks = None
    sampler = None
    if rank == 0:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        sampler.start()
        time.sleep(0.05)

    # -- timed region A: the product call, back to back -------------------
    launches = 0  # kernels of this library launched in region A
    mark_a = sampler.mark() if sampler else 0
    barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        step(Xs[i % n_copies])
        launches += kernels_per_step
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    step_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps)
    mark_a_end = sampler.mark() if sampler else 0

    # -- timed region B: each pass alone, back to back (kernel durations) --
    # K launches of the fused pass between two events on its stream, then K
    # launches of the finalize pass; the mean duration of a launch is the
    # span over K.  Back to back, a launch's set-up overlaps the end of the
    # one before (programmatic dependent launch), as in region A.
    def time_pass(fn):
        ea = torch.cuda.Event(enable_timing=True)
        eb = torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(dev)
        ea.record(stream)
        for i in range(args.steps):
            fn(Xs[i % n_copies])
        eb.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        return max_over_ranks(ea.elapsed_time(eb) / args.steps)

    fused_ms = time_pass(first_pass)
    fin_ms = time_pass(lambda x: q.finalize(x, offsets, Xt, m, ws, stream=stream))
    if read_device_status(ws, stream) != 0:
        raise RuntimeError("device flags raised during the timed region")

    # -- timed region C: end to end on host buffers ----------------------
    X_host = X.cpu().pin_memory()
    offs_host = np.ascontiguousarray(inp["offsets"])
    out_x = torch.empty((B, w.k, w.d), dtype=torch.float32).pin_memory()
    out_m = torch.empty((B, w.k), dtype=torch.float32).pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    if uq:
        # Per-user queries have no host-buffer entry point: pinned host
        # copies of X, the offsets and the queries on the same stream, the
        # device call, and the copies of the results back.
        offs_pinned = torch.from_numpy(offs_host).pin_memory()
        X_e, off_e, Q_e = torch.empty_like(X), torch.empty_like(offsets), torch.empty_like(Qd)

        def e2e_step():
            X_e.copy_(X_host, non_blocking=True)
            off_e.copy_(offs_pinned, non_blocking=True)
            Q_e.copy_(Q_host, non_blocking=True)
            q.forward_user_queries(Q_e, X_e, off_e, Xt, m, ws, stream=stream)
            out_x.copy_(Xt, non_blocking=True)
            out_m.copy_(m, non_blocking=True)
    else:
        dev_buf = torch.empty(q.host_path_device_bytes(B, N), dtype=torch.uint8, device=dev)
        ox, om = out_x.numpy(), out_m.numpy()

        def e2e_step():
            q.forward_host(X_host, offs_host, dev_buf, stream=stream, out_x=ox, out_m=om)
    e2e_step()
    barrier()
    torch.cuda.synchronize(dev)
    h0 = torch.cuda.Event(enable_timing=True)
    h1 = torch.cuda.Event(enable_timing=True)
    h0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    h1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(h0.elapsed_time(h1) / e2e_steps)

    # -- region D: sustained, back to back for about args.sustained seconds --
    sustained = None
    if args.sustained > 0:
        mark_d = sampler.mark() if sampler else 0
        n_sus = max(args.steps, int(args.sustained / max(step_ms * 1e-3, 1e-6)))
        barrier()
        torch.cuda.synchronize(dev)
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for i in range(n_sus):
            step(Xs[i % n_copies])
        s1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        sus_ms = max_over_ranks(s0.elapsed_time(s1) / n_sus)
        sustained = {"ms_per_step": sus_ms, "steps": n_sus,
                     "seconds": sus_ms * n_sus * 1e-3,
                     "value": ranks.sum(N) / (sus_ms * 1e-3),
                     "clocks": sampler.summary(mark_d) if sampler else None}

    if sampler is not None:
        sampler.stop()
        # the kernel-only regions A and B (region C is mostly host copies)
        clocks = sampler.summary(mark_a, mark_a_end) or sampler.summary(mark_a)

    # sanity on the last outputs: every behaviour spreads unit mass
    msum = m.sum(dim=1).double().cpu().numpy()
    n_b = np.diff(inp["offsets"]).astype(np.float64)
    if np.max(np.abs(msum - n_b) / np.maximum(n_b, 1)) > 1e-3:
        raise RuntimeError("mass check failed")

    if rank != 0:
        return
    peaks, peak_kind = load_peaks()
    bytes_x = float(N) * w.d * elem
    flops = 4.0 * w.k * w.d * N
    t_hbm = bytes_x / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    fused_s = fused_ms * 1e-3
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    if bound == "hbm":
        achieved, peak, unit = bytes_x / fused_s / 1e9, peaks["hbm_gbs"], "GB/s"
    else:
        achieved, peak, unit = flops / fused_s / 1e12, peaks["bf16_tflops"], "TFLOP/s"
    traffic = None if uq else load_traffic(args.workload)  # captures cover shared queries
    rows_total = ranks.sum(N)  # rows of all ranks' batches
    value = rows_total / (step_ms * 1e-3)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        rps, rows, dt, users = oracle_rows_per_s(inp, args.cpu_budget,
                                                 queries=Q_host.numpy() if uq else None)
        cpu = {"value": rps, "unit": "rows/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"users {users[0]}..{users[-1]} ({rows} rows, {dt:.1f} s, numpy fp64)"}
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "rows/s",
        "n_gpus": args.gpus,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": step_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": {
            "workload": args.workload, "users_per_gpu": B, "rows_per_gpu": N,
            "d": w.d, "k": w.k, "x_bytes_per_gpu": bytes_x,
            "l2": (f"inputs larger than L2 (X {bytes_x / 1e6:.1f} MB > {L2_BYTES / 1e6:.0f} MB)"
                   if n_copies == 1 else
                   f"X {bytes_x / 1e6:.1f} MB fits in L2: timed iterations rotate over "
                   f"{n_copies} copies ({n_copies * bytes_x / 1e6:.0f} MB > 2 x L2)"),
            "parallelism": f"independent batch per GPU x{world}",
            "queries": ("per user: B x k x d fp32, the SA step of a refinement layer"
                        if uq else "shared prototypes P"),
        },
        "roofline": {
            "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
            "frac": achieved / peak, "traffic": traffic,
            "kernel": ("user_query_kernel + " if uq else "") +
                      ("simt_fp32_kernel" if w.dtype != "bf16" else
                       "fused_sa_pair_kernel" if w.d == 256 and w.k > 64 else
                       f"fused_sa_kernel<{w.d},128> on clusters of {-(-w.k // 128)} CTAs"
                       if w.k > 128 else
                       f"fused_sa_kernel<{w.d},{64 if w.k <= 64 else 128}>"),
            "kernel_ms": fused_ms, "finalize_ms": fin_ms,
            "kernel_timing": f"mean over {args.steps} back-to-back launches of the pass, "
                             "CUDA events on its stream",
            "roofline_ms": 1e3 * max(t_hbm, t_tc),
            "tensor_frac": (flops / fused_s / 1e12) / peaks["bf16_tflops"],
            "hbm_frac": (bytes_x / fused_s / 1e9) / peaks["hbm_gbs"],
            "peak_source": f"MEASURED_PEAKS.json ({peak_kind}, burst)",
            "algorithmic": f"{2 * w.d} B and {4 * w.k * w.d} flop per row x {N} rows",
        },
        "e2e": {"value": rows_total / (e2e_ms * 1e-3), "unit": "rows/s",
                "h2d_bytes_per_step": int(bytes_x + 8 * (B + 1) + (4 * B * w.k * w.d if uq else 0)),
                "d2h_bytes_per_step": int(4 * B * w.k * (w.d + 1)),
                "ms_per_step": e2e_ms},
        "gpu_launches": launches,
        "clocks": clocks,
        "sustained": sustained,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def _timed(fn, steps, dev, stream, ranks):
    """Mean ms of `steps` back-to-back calls of fn between two CUDA events on
    `stream`, bracketed by barrier + synchronize; max over ranks."""
    import torch
    ranks.barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ranks.barrier()
    return ranks.max(e0.elapsed_time(e1) / steps)


def _roofline(bytes_per_launch, flops_per_launch, ms, peaks, peak_kind, kernel, note):
    t_hbm = bytes_per_launch / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops_per_launch / (peaks["bf16_tflops"] * 1e12)
    s = ms * 1e-3
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    if bound == "hbm":
        achieved, peak, unit = bytes_per_launch / s / 1e9, peaks["hbm_gbs"], "GB/s"
    else:
        achieved, peak, unit = flops_per_launch / s / 1e12, peaks["bf16_tflops"], "TFLOP/s"
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
            "frac": achieved / peak, "traffic": None, "kernel": kernel, "kernel_ms": ms,
            "roofline_ms": 1e3 * max(t_hbm, t_tc),
            "tensor_frac": (flops_per_launch / s / 1e12) / peaks["bf16_tflops"],
            "hbm_frac": (bytes_per_launch / s / 1e9) / peaks["hbm_gbs"],
            "peak_source": f"MEASURED_PEAKS.json ({peak_kind}, burst)", "algorithmic": note}


def run_backward(args, rank, world, local_rank, ranks):
    """One step = sa_sketch_backward over the batch (upstream gradients G, g
    seeded), the SA backward of section 2.2's end-to-end training."""
    import torch

    from sketch_attention_compression_b200 import SketchQuery, load_library, read_device_status
    from synthetic import upstream_gradients
    load_library()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = WORKLOADS[args.workload]
    inp = workload_inputs(args, seed=rank_seed(args.workload, rank))
    X = torch.from_numpy(inp["X"]).to(dev).to(torch.bfloat16)
    P, W_Q, W_K = (torch.from_numpy(inp[k]).to(dev).to(torch.bfloat16) for k in ("P", "W_Q", "W_K"))
    f32 = {k: torch.from_numpy(inp[k]).to(dev) for k in ("P", "W_Q", "W_K")}
    offsets = torch.from_numpy(inp["offsets"]).to(dev)
    B, N = len(inp["offsets"]) - 1, int(inp["offsets"][-1])
    Gn, gn = upstream_gradients(B, w.k, w.d, seed=rank_seed(args.workload, rank) + 200)
    G = torch.from_numpy(Gn.astype(np.float32)).to(dev)
    g = torch.from_numpy(gn.astype(np.float32)).to(dev)
    stream = torch.cuda.current_stream(dev)
    q = SketchQuery(P, W_Q, W_K, inp["scale"], stream=stream)
    _, ws = q.backward(X, offsets, G, g, P_f32=f32["P"], W_Q_f32=f32["W_Q"], W_K_f32=f32["W_K"])

    def step():
        q.backward(X, offsets, G, g, P_f32=f32["P"], W_Q_f32=f32["W_Q"], W_K_f32=f32["W_K"],
                   workspace=ws, stream=stream)
    for _ in range(args.warmup):
        step()
    if read_device_status(ws, stream) != 0:
        raise RuntimeError("device flags raised during warm-up")
    sampler = None
    if rank == 0:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        sampler.start()
        time.sleep(0.05)
    mark = sampler.mark() if sampler else 0
    ms = _timed(step, args.steps, dev, stream, ranks)
    clocks = sampler.summary(mark) if sampler else None
    if sampler:
        sampler.stop()
    if read_device_status(ws, stream) != 0:
        raise RuntimeError("device flags raised during the timed region")
    if rank != 0:
        return
    peaks, peak_kind = load_peaks()
    rows_total = ranks.sum(N)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        from oracle import sa_user_backward
        t0 = time.perf_counter()
        rows, done = 0, 0
        offs = inp["offsets"]
        for b in range(B):
            lo, hi = int(offs[b]), int(offs[b + 1])
            sa_user_backward(inp["X"][lo:hi], inp["P"], inp["W_Q"], inp["W_K"], inp["scale"],
                             Gn[b], gn[b])
            rows += hi - lo
            done = b
            if time.perf_counter() - t0 >= args.cpu_budget:
                break
        dt = time.perf_counter() - t0
        cpu = {"value": rows / dt, "unit": "rows/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"users 0..{done} ({rows} rows, {dt:.1f} s, numpy fp64 sa_user_backward)"}
    line = {
        "metric": "SA backward history rows/sec on 1 B200 (dX, dP, dW_Q, dW_K)",
        "value": rows_total / (ms * 1e-3), "unit": "rows/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "mode": "backward", "users_per_gpu": B,
                   "rows_per_gpu": N, "d": w.d, "k": w.k, "upstream": "G, g ~ N(0, 1)"},
        "roofline": _roofline(4.0 * w.d * N, 10.0 * w.k * w.d * N, ms, peaks, peak_kind,
                              "sa_sketch_backward (prep + backward pass + finalize + GEMMs)",
                              f"{4 * w.d} B (X read, dX written) and {10 * w.k * w.d} flop "
                              f"per row x {N} rows"),
        "clocks": clocks, "cpu_baseline": cpu,
        "gpu_launches": None,
    }
    print(json.dumps(line), flush=True)


def run_refine(args, rank, world, local_rank, ranks):
    """One step = sa_refine_stack_forward with --refine-layers layers over the
    batch (section 2.2's stacked refinement; each layer one SA pass over X
    plus the LN / SwiGLU update of the B x k sketches)."""
    import torch

    from sketch_attention_compression_b200 import (RefineParams, SketchQuery, load_library,
                                                   read_device_status, refine_stack_forward)
    from synthetic import refine_params
    load_library()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = WORKLOADS[args.workload]
    L, h = args.refine_layers, 4 * w.d
    inp = workload_inputs(args, seed=rank_seed(args.workload, rank))
    X = torch.from_numpy(inp["X"]).to(dev).to(torch.bfloat16)
    offsets = torch.from_numpy(inp["offsets"]).to(dev)
    B, N = len(inp["offsets"]) - 1, int(inp["offsets"][-1])
    P = torch.from_numpy(inp["P"]).to(dev)
    stream = torch.cuda.current_stream(dev)
    qs, rs = [], []
    for layer in range(L):
        p = refine_params(w.d, h, seed=rank_seed(args.workload, rank) + 300 + layer)
        qs.append(SketchQuery(P.to(torch.bfloat16), torch.from_numpy(p["W_Q"]).to(dev).to(torch.bfloat16),
                              torch.from_numpy(p["W_K"]).to(dev).to(torch.bfloat16), p["scale"],
                              stream=stream))
        t = {key: torch.from_numpy(p[key]).to(dev) for key in ("W1", "W3", "W2", "gamma1", "beta1",
                                                                 "gamma2", "beta2")}
        rs.append(RefineParams(t["W1"], t["W3"], t["W2"], t["gamma1"], t["beta1"], t["gamma2"],
                               t["beta2"], stream=stream))
    out, ws = refine_stack_forward(qs, rs, P, X, offsets, stream=stream)

    def step():
        refine_stack_forward(qs, rs, P, X, offsets, out=out, workspace=ws, stream=stream)
    for _ in range(args.warmup):
        step()
    if read_device_status(ws, stream) != 0:
        raise RuntimeError("device flags raised during warm-up")
    sampler = None
    if rank == 0:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        sampler.start()
        time.sleep(0.05)
    mark = sampler.mark() if sampler else 0
    ms = _timed(step, args.steps, dev, stream, ranks)
    clocks = sampler.summary(mark) if sampler else None
    if sampler:
        sampler.stop()
    if read_device_status(ws, stream) != 0:
        raise RuntimeError("device flags raised during the timed region")
    if rank != 0:
        return
    peaks, peak_kind = load_peaks()
    rows_total = ranks.sum(N)
    flops = L * (4.0 * w.k * w.d * N + 6.0 * h * w.d * B * w.k)
    line = {
        "metric": f"SA refinement stack ({L} layers) history rows/sec on 1 B200",
        "value": rows_total / (ms * 1e-3), "unit": "rows/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "mode": f"refine_stack x{L}", "users_per_gpu": B,
                   "rows_per_gpu": N, "d": w.d, "k": w.k, "ffn_hidden": h},
        "roofline": _roofline(L * 2.0 * w.d * N, flops, ms, peaks, peak_kind,
                              "sa_refine_stack_forward (per layer: SA pass + finalize + update)",
                              f"per layer {2 * w.d} B and {4 * w.k * w.d} flop per row x {N} rows, "
                              f"plus 6 h d flop per (user, prototype) row"),
        "clocks": clocks, "cpu_baseline": None, "gpu_launches": None,
    }
    print(json.dumps(line), flush=True)


def run_action(args, rank, world, local_rank, ranks):
    """One step = sa_action_sketch_forward over the batch: the action-fusion
    producer X = E + SwiGLU-FFN([E; a]) (section 2.2, hidden width
    --action-hidden, four action types) followed by the SA layer on X."""
    import torch

    from sketch_attention_compression_b200 import (ActionFusion, SketchQuery, load_library,
                                                   read_device_status)
    from synthetic import action_params, action_types
    load_library()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = WORKLOADS[args.workload]
    h, n_types = args.action_hidden, 4
    seed = rank_seed(args.workload, rank)
    inp = workload_inputs(args, seed=seed)
    B, N = len(inp["offsets"]) - 1, int(inp["offsets"][-1])
    E = torch.from_numpy(inp["X"]).to(dev).to(torch.bfloat16)
    types_np = action_types(N, n_types, seed=seed + 400)
    types = torch.from_numpy(types_np).to(dev)
    offsets = torch.from_numpy(inp["offsets"]).to(dev)
    p = action_params(w.d, w.d, h, n_types, seed=seed + 401)
    stream = torch.cuda.current_stream(dev)
    t = {key: torch.from_numpy(p[key]).to(dev) for key in ("W1", "W3", "W2", "table")}
    act = ActionFusion(t["W1"], t["W3"], t["W2"], t["table"], stream=stream)
    q = SketchQuery(*(torch.from_numpy(inp[k]).to(dev).to(torch.bfloat16) for k in ("P", "W_Q", "W_K")),
                    inp["scale"], stream=stream)
    Xt, m, ws = act.sketch_forward(q, E, types, offsets, stream=stream)
    Xbuf = torch.empty_like(E)

    def step():
        act.sketch_forward(q, E, types, offsets, X_tilde=Xt, mass=m, workspace=ws, stream=stream)

    def producer():
        act.fuse(E, types, out=Xbuf, stream=stream)
    for _ in range(args.warmup):
        step()
        producer()
    if read_device_status(ws, stream) != 0:
        raise RuntimeError("device flags raised during warm-up")
    sampler = None
    if rank == 0:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        sampler.start()
        time.sleep(0.05)
    mark = sampler.mark() if sampler else 0
    ms = _timed(step, args.steps, dev, stream, ranks)
    ms_prod = _timed(producer, args.steps, dev, stream, ranks)
    clocks = sampler.summary(mark) if sampler else None
    if sampler:
        sampler.stop()
    if read_device_status(ws, stream) != 0:
        raise RuntimeError("device flags raised during the timed region")
    if rank != 0:
        return
    peaks, peak_kind = load_peaks()
    rows_total = ranks.sum(N)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        from oracle import action_fuse, sa_user
        t0 = time.perf_counter()
        rows, done = 0, 0
        offs = inp["offsets"]
        for b in range(B):
            lo, hi = int(offs[b]), int(offs[b + 1])
            Xo = action_fuse(inp["X"][lo:hi], types_np[lo:hi], p["table"], p["W1"], p["W3"], p["W2"])
            sa_user(Xo, inp["P"], inp["W_Q"], inp["W_K"], inp["scale"])
            rows += hi - lo
            done = b
            if time.perf_counter() - t0 >= args.cpu_budget:
                break
        dt = time.perf_counter() - t0
        cpu = {"value": rows / dt, "unit": "rows/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"users 0..{done} ({rows} rows, {dt:.1f} s, numpy fp64 action_fuse + sa_user)"}
    line = {
        "metric": "action fusion + SA history rows/sec on 1 B200",
        "value": rows_total / (ms * 1e-3), "unit": "rows/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "mode": "action_fusion + sa", "users_per_gpu": B,
                   "rows_per_gpu": N, "d": w.d, "k": w.k, "ffn_hidden": h, "action_types": n_types,
                   "action_width": w.d, "producer_ms": ms_prod},
        "roofline": _roofline((4.0 * w.d + 1.0) * N, 6.0 * w.d * h * N, ms_prod, peaks, peak_kind,
                              "action_fuse_kernel (the producer alone)",
                              f"{6 * w.d * h} flop (E W1, E W3, G W2; the action term is a "
                              f"per-type row) and {4 * w.d + 1} B (E read, X written, type) "
                              f"per row x {N} rows"),
        "clocks": clocks, "cpu_baseline": cpu,
        "gpu_launches": 3 * args.steps + args.steps,
    }
    print(json.dumps(line), flush=True)


def run_cache(args, rank, world, local_rank, ranks):
    """The sketch cache on the workload (section 2.4): one step = one SA layer
    served through sa_cache_forward for every user of the batch, at a fixed
    group hit rate (the notes report about 0.6 in serving with a one-hour
    TTL and 0.5 in training with three hours).  The hit users keep their
    keys; the others arrive with a new history timestamp each step, so they
    miss, are compressed from their rows and inserted.  Also timed: all
    hits, all misses, and the width adapter (D = 1024) on the batch's
    sketches."""
    import torch

    from sketch_attention_compression_b200 import (SketchCache, SketchQuery, WidthAdapter,
                                                   load_library)
    load_library()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = WORKLOADS[args.workload]
    inp = workload_inputs(args, seed=rank_seed(args.workload, rank))
    B, N = len(inp["offsets"]) - 1, int(inp["offsets"][-1])
    X = torch.from_numpy(inp["X"]).to(dev).to(torch.bfloat16)
    stream = torch.cuda.current_stream(dev)
    q = SketchQuery(*(torch.from_numpy(inp[k]).to(dev).to(torch.bfloat16) for k in ("P", "W_Q", "W_K")),
                    inp["scale"], stream=stream)
    offsets_host = np.ascontiguousarray(inp["offsets"], dtype=np.int64)
    Xt = torch.empty((B, w.k, w.d), dtype=torch.float32, device=dev)
    m = torch.empty((B, w.k), dtype=torch.float32, device=dev)
    total_steps = 4 * (args.warmup + args.steps) + 8
    cache = SketchCache(w.k, w.d, capacity=B * (total_steps + 2), ttl=3600.0)
    ws = None
    clock = [0.0]
    ts_counter = [1000]

    def make_step(hit_rate):
        n_hit = int(round(hit_rate * B))
        # (user, model version, history timestamp, config) per user
        keys = np.array([(rank * 100000 + b, 1, 0, 7) for b in range(B)], dtype=np.int64)

        def step():
            nonlocal ws
            clock[0] += 0.001
            ts_counter[0] += 1
            keys[n_hit:, 2] = ts_counter[0]  # the misses: a new history timestamp
            _, _, hit, ws = cache.forward(q, keys, clock[0], X, offsets_host, X_tilde=Xt, mass=m,
                                          workspace=ws, stream=stream)
            return hit
        return step, n_hit

    timings = {}
    for name, rate in (("hit_0.6", 0.6), ("hit_0.5", 0.5), ("all_hits", 1.0), ("all_misses", 0.0)):
        step, n_hit = make_step(rate)
        for _ in range(args.warmup):
            hit = step()
        assert int(hit.sum()) == n_hit, (name, int(hit.sum()), n_hit)
        timings[name] = _timed(step, args.steps, dev, stream, ranks)
    rng = np.random.default_rng(7)
    W_A = torch.from_numpy((rng.standard_normal((w.d, 1024)) / np.sqrt(w.d)).astype(np.float32)).to(dev)
    ad = WidthAdapter(W_A, stream=stream)
    Y = ad.forward(Xt.reshape(-1, w.d), stream=stream)

    def adapt():
        ad.forward(Xt.reshape(-1, w.d), out=Y, stream=stream)
    for _ in range(args.warmup):
        adapt()
    ms_adapter = _timed(adapt, args.steps, dev, stream, ranks)
    if rank != 0:
        return
    ms = timings["hit_0.6"]
    peaks, _ = load_peaks()
    rows_ad = B * w.k
    line = {
        "metric": "users served per second through the sketch cache at a 0.6 hit rate",
        "value": ranks.sum(B) / (ms * 1e-3), "unit": "users/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "mode": "sketch cache", "users_per_gpu": B,
                   "rows_per_gpu": N, "d": w.d, "k": w.k,
                   "ms_per_step_by_hit_rate": {k: round(v, 4) for k, v in timings.items()},
                   "adapter": {"rows": rows_ad, "D": 1024, "ms": round(ms_adapter, 4),
                               "tflops": 2.0 * w.d * 1024 * rows_ad / (ms_adapter * 1e-3) / 1e12,
                               "frac_of_bf16_peak": 2.0 * w.d * 1024 * rows_ad /
                               (ms_adapter * 1e-3) / 1e12 / peaks["bf16_tflops"]}},
        "roofline": None,
        "note": ("a composed path (host index, host-to-device slot lists, gather, SA pass over "
                 "the missed users' rows, scatter): its kernels' rooflines are on the SA lines; "
                 "the adapter is a few-microsecond GEMM"),
        "clocks": None, "cpu_baseline": None, "gpu_launches": None,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--cpu-budget", type=float, default=10.0,
                    help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--user-queries", action="store_true",
                    help="query every user with its own k x d matrix (refinement-layer SA step)")
    ap.add_argument("--sustained", type=float, default=2.0,
                    help="seconds of back-to-back whole steps after the timed regions, reported "
                         "as 'sustained' with their own clocks (0: skip)")
    ap.add_argument("--backward", action="store_true",
                    help="time the SA backward pass (sa_sketch_backward) instead")
    ap.add_argument("--refine-layers", type=int, default=0,
                    help="time a stack of this many refinement layers instead")
    ap.add_argument("--cache", action="store_true",
                    help="time the layer served through the sketch cache (and the width adapter)")
    ap.add_argument("--action-fusion", action="store_true",
                    help="time the action-fusion producer followed by the SA layer instead")
    ap.add_argument("--action-hidden", type=int, default=512,
                    help="hidden width of the action-fusion FFN")
    ap.add_argument("--users", type=int, default=0,
                    help="use only the first U users of the workload (smaller case)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if world != args.gpus:
        # One process per GPU: N GPUs need N ranks (torchrun --nproc-per-node
        # N).  A mismatch would time a different number of GPUs than the line
        # reports.
        ap.error(f"--gpus {args.gpus} but {world} rank(s) were launched "
                 "(use torchrun --nproc-per-node N for N > 1)")
    if args.impl == "reference":
        run_reference(args, rank)
        return
    ranks = init_rank_group(world, local_rank, "nccl")
    try:
        if args.backward:
            run_backward(args, rank, world, local_rank, ranks)
        elif args.refine_layers > 0:
            run_refine(args, rank, world, local_rank, ranks)
        elif args.action_fusion:
            run_action(args, rank, world, local_rank, ranks)
        elif args.cache:
            run_cache(args, rank, world, local_rank, ranks)
        else:
            run_ours(args, rank, world, local_rank, ranks)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
