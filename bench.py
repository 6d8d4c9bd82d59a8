#!/usr/bin/env python3
"""Benchmark: exact attention forward TFLOP/s on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one exact-attention forward (one launch of the C entry point fa_fwd:
the "auto" schedule picks the static schedule for this size; --schedule
dynamic times fa_fwd_dynamic) over
one batch of the long-context causal workload (B=2, H=32, N=8192, d=128, bf16, seeded
N(0,1) inputs), inputs resident in HBM.  FLOPs per step: 4*B*H*N^2*d / 2.
Prints one JSON line (rank 0).

For N > 1 (torchrun, one process per GPU) every rank runs its own batch of
the same shape: the forward has no exchange step, so the ranks share nothing
but the barrier and the max-over-ranks timing reduction (weak scaling).

``--impl reference`` times the fp64 CPU oracle on the host cores instead (the
reference arm): each step is a bounded sample of the same workload.

``--decode`` instead times the decode-shaped path (fa_fwd_decode: 1 new
query per sequence against 32K keys, B=16, H=32, d=128), which is bound by
reading K and V once: its metric is effective HBM GB/s.

``--sweep`` instead prints one line per sequence length of the page's
"Try It Yourself" sweep (B=1, H=32, d=128, causal, N = 512..8192), device
timed like the main line; it is an extra curve, not the headline number.

A workload whose step moves less than twice the 126 MB L2 (``--workload``
1-3, the sweep below N = 8192) is timed differently: the launches cycle
through enough copies of the buffers that none finds its inputs in L2, L2
is flushed before the timed region, and the launches are replayed from one
CUDA graph, since eager launches of a few microseconds would time the host.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "attention fwd TFLOP/s and % of B200 dense BF16 peak (1 GPU)"
UNIT = "TFLOP/s"
WORKLOAD_INDEX = 4          # long-context causal: B=2, H=32, N=8192, d=128
KERNEL_SOURCE = os.path.join(ROOT, "exact_attention_122_b200", "csrc", "fa_fwd_sm100.cu")
BWD_KERNEL_SOURCE = os.path.join(ROOT, "exact_attention_122_b200", "csrc", "fa_bwd_sm100.cu")
DECODE_KERNEL_SOURCE = os.path.join(ROOT, "exact_attention_122_b200", "csrc", "fa_decode_sm100.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAK_TFLOPS = 1590.0   # used only when the measured peaks file is absent
# NVIDIA's dense BF16 figure for one B200 (half its 2:4-sparse 4.5 PFLOP/s), reported beside the
# measured peak for context; the roofline fraction uses the measured one.
NOMINAL_BF16_TFLOPS = 2250.0


# ---------------------------------------------------------------------------
# Host-side helpers (also exercised by the CPU tests)
# ---------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return world, rank, local


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own batch (independent problems, weak scaling)."""
    return base_seed + 1000 * rank


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank float over the process group (identity if none)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sample_plan(w: synth.Workload, rows: int):
    """Bounded oracle sample: the last ``rows`` query rows of head 0 (the
    rows with the most allowed keys).  Returns (row indices, FLOPs)."""
    rows = max(1, min(rows, w.N))
    idx = list(range(w.N - rows, w.N))
    if w.causal:
        keys = sum(i + 1 for i in idx)
    else:
        keys = rows * w.N
    return idx, 4.0 * keys * w.d


def kernel_source_sha(path: str = KERNEL_SOURCE) -> str:
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", 0.0)), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_PEAK_TFLOPS, 0.0, "fallback"


def load_traffic(workload_name: str, source: str = KERNEL_SOURCE):
    """Per-launch DRAM bytes of the dominant kernel from the committed ncu
    summaries, only while that kernel's source file still matches the one
    that was profiled.  The file holds {"entries": [...]}, each entry naming
    its workload, its kernel source (relative to the repository) and that
    source's sha256."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    entries = t.get("entries", [t]) if isinstance(t, dict) else []
    rel = os.path.relpath(source, ROOT)
    for e in entries:
        if e.get("workload") != workload_name:
            continue
        if e.get("kernel_source", os.path.relpath(KERNEL_SOURCE, ROOT)) != rel:
            continue
        if e.get("kernel_source_sha256") != kernel_source_sha(source):
            return None
        return e.get("bytes_per_launch")
    return None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x0000000000000004: "sw_power_cap",
        0x0000000000000008: "hw_slowdown",
        0x0000000000000020: "sw_thermal_slowdown",
        0x0000000000000040: "hw_thermal_slowdown",
        0x0000000000000080: "hw_power_brake_slowdown",
        0x0000000000000010: "sync_boost",
        0x0000000000000100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.ok = False
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            uuid = None
            try:
                import torch
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            except Exception:
                pass
            self._h = None
            if uuid:
                try:
                    self._h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
                except Exception:
                    self._h = None
            if self._h is None:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "source": "nvml unavailable" if not self.ok else "no samples"}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml"}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        info = threadpool_info()
        return max((i.get("num_threads", 0) for i in info), default=0)
    except Exception:
        return 0


def time_oracle_sample(w: synth.Workload, q, k, v, target_s: float):
    """Time the fp64 oracle on a bounded sample of the workload.

    The sample grows from the last rows of head 0 (the rows with the most
    allowed keys) to whole heads 0, 1, 2, ... until it has taken about
    ``target_s`` seconds.  Returns (TFLOP/s, seconds, description)."""
    import numpy as np

    import oracle

    BH = w.B * w.H
    q3, k3, v3 = (t.reshape(BH, w.N, w.d) for t in (q, k, v))
    head = lambda h: tuple(oracle.exact_attention._as_f64(t[h]) for t in (q3, k3, v3))
    qb, kb, vb = head(0)
    rows = 64
    while True:
        idx, flops = sample_plan(w, rows)
        t0 = time.perf_counter()
        oracle.attention_rows_fp64(qb, kb, vb, np.array(idx), w.causal, w.scale)
        dt = time.perf_counter() - t0
        if dt >= target_s or rows >= w.N:
            break
        rows = min(w.N, int(rows * max(2.0, min(16.0, target_s / max(dt, 1e-3)))))
    total_flops, total_dt, heads = flops, dt, 1
    while total_dt < target_s and heads < BH:
        qb, kb, vb = head(heads)
        idx, flops = sample_plan(w, w.N)
        t0 = time.perf_counter()
        oracle.attention_rows_fp64(qb, kb, vb, np.array(idx), w.causal, w.scale)
        total_dt += time.perf_counter() - t0
        total_flops += flops
        heads += 1
    if heads == 1:
        what = f"the last {rows} query rows of head 0"
    else:
        what = f"all rows of heads 0..{heads - 1}"
    desc = (f"fp64 oracle (materialised S and P rows) on {what} of {w.describe()}, "
            f"{total_flops / 1e9:.1f} GFLOP")
    return total_flops / total_dt / 1e12, total_dt, desc


# ---------------------------------------------------------------------------
# Reference arm: the oracle on the host cores
# ---------------------------------------------------------------------------

def run_reference(args, w):
    world, rank, _ = dist_env()
    if world > 1 and rank != 0:
        return 0
    import numpy as np

    import oracle

    q, k, v = synth.workload_qkv(w)
    qb, kb, vb = (oracle.exact_attention._as_f64(t[0, 0]) for t in (q, k, v))
    steps_total = args.steps + args.warmup
    per_step = max(0.05, min(2.0, 150.0 / max(1, steps_total)))
    # calibrate the row count for ~per_step seconds
    rows = 32
    while True:
        idx, flops = sample_plan(w, rows)
        t0 = time.perf_counter()
        oracle.attention_rows_fp64(qb, kb, vb, np.array(idx), w.causal, w.scale)
        dt = time.perf_counter() - t0
        if dt >= per_step * 0.7 or rows >= w.N:
            break
        rows = min(w.N, int(rows * max(1.5, min(8.0, per_step / max(dt, 1e-4)))))
    idx, flops = sample_plan(w, rows)
    idx = np.array(idx)
    for _ in range(args.warmup):
        oracle.attention_rows_fp64(qb, kb, vb, idx, w.causal, w.scale)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.attention_rows_fp64(qb, kb, vb, idx, w.causal, w.scale)
    dt = time.perf_counter() - t0
    value = flops * args.steps / dt / 1e12
    cores = blas_threads() or os.cpu_count()
    sample = (f"each step: fp64 oracle on the last {len(idx)} query rows of head 0 of "
              f"{w.describe()} ({flops / 1e9:.2f} GFLOP)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, args.gpus, bench_schedule(args.schedule, w),
                                  1 if args.l2_warm else rotation_copies(w.algorithmic_bytes,
                                                                         args.steps),
                                  args.l2_warm),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


L2_BYTES = 126 * 1000 * 1000    # B200 L2 capacity


def rotation_copies(step_bytes: int, steps: int) -> int:
    """Copies of one step's buffers that the timed launches cycle through so
    that no launch finds its inputs in L2: 1 when a step alone moves at least
    twice the L2 capacity; otherwise enough copies that at least twice the L2
    capacity streams between two uses of one copy, but never more copies than
    launches (each copy is then used once, after an L2 flush)."""
    if step_bytes >= 2 * L2_BYTES:
        return 1
    return max(2, min(steps, math.ceil(2 * L2_BYTES / step_bytes) + 1))


def l2_note(step_bytes: int, copies: int, warm: bool = False) -> str:
    if warm:
        return (f"L2-warm on purpose (--l2-warm): one step moves {step_bytes / 1e6:.1f} MB, one set "
                f"of buffers reused, no flush; launches replayed from one CUDA graph")
    if copies == 1:
        return f"one step moves {step_bytes / 1e6:.0f} MB > 2 x 126 MB L2; no flush"
    return (f"one step moves {step_bytes / 1e6:.1f} MB < 2 x 126 MB L2: launches cycle through "
            f"{copies} copies of the buffers and L2 is flushed (252 MB write) before the timed "
            f"region; launches replayed from one CUDA graph")


B200_SM_COUNT = 148


def bench_schedule(schedule: str, w: synth.Workload, sm_count: int | None = None) -> str:
    """The forward schedule a line uses ("auto" resolved the way fa_fwd
    resolves it; the reference arm, which needs no GPU, assumes a B200)."""
    from exact_attention_122_b200._binding import resolve_schedule

    return resolve_schedule(schedule, w.B, w.H, w.N, sm_count or B200_SM_COUNT)


def require_beyond_l2(step_bytes: int, steps: int, mode: str) -> None:
    """The --bwd and --fp8 lines time eager launches without an L2 flush, which
    is valid only when one step moves at least twice the L2 capacity."""
    if rotation_copies(step_bytes, steps) != 1:
        raise SystemExit(f"{mode} times workloads whose step moves >= {2 * L2_BYTES / 1e6:.0f} MB "
                         f"(this one moves {step_bytes / 1e6:.1f} MB): use --workload 4 or 5")


def fwd_kernel_name(d: int, fp8: bool = False) -> str:
    ns = {(128, False): 4, (64, False): 8, (128, True): 8, (64, True): 16}[(d, fp8)]
    return f"fa_fwd_kernel<{d},{ns}{',true' if fp8 else ''}>"


def time_graph(launch, n_launch: int, replays: int, stream, local: int, sync_all,
               flush_l2: bool = True):
    """Capture launch(0..n_launch-1) into one CUDA graph, replay it once
    untimed, flush L2 (unless flush_l2 is False), then time `replays`
    replays with CUDA events on `stream`.  Returns (total ms, clock summary)."""
    import torch

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(n_launch):
            launch(i)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=stream.device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        g.replay()
        if flush_l2:
            flush.zero_()
    sync_all()
    with ClockSampler(local) as clocks:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(replays):
                g.replay()
            e1.record(stream)
        sync_all()
    total = e0.elapsed_time(e1)
    del g
    return total, clocks.summary()


def workload_config(w: synth.Workload, n_gpus: int, schedule: str = "dynamic", copies: int = 1,
                    warm: bool = False):
    return {"workload": w.name, "schedule": schedule,
            "B_per_gpu": w.B, "H": w.H, "N": w.N, "d": w.d,
            "causal": w.causal, "scale": w.scale, "global_batch": w.B * n_gpus, "seq_len": w.N,
            "parallelism": f"independent batches x{n_gpus}" if n_gpus > 1 else "single GPU",
            "l2": l2_note(w.algorithmic_bytes, copies, warm)}


# ---------------------------------------------------------------------------
# Our arm
# ---------------------------------------------------------------------------

def run_ours(args, w):
    import torch
    import torch.distributed as dist

    import exact_attention_122_b200 as fa

    world, rank, local = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    sched = bench_schedule(args.schedule, w, torch.cuda.get_device_properties(dev).multi_processor_count)
    q, k, v = synth.draw_qkv(w.B, w.H, w.N, w.d, rank_seed(w.seed, rank), w.qk_std)
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    od = torch.empty_like(qd)
    lsed = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step():
        fa.fa_fwd(qd, kd, vd, causal=w.causal, scale=w.scale, out=od, lse=lsed, stream=stream,
                  schedule=sched)

    def sync_all():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    st, word = fa.device_status(stream.cuda_stream)
    if st != fa.FA_OK:
        raise SystemExit(f"kernel status {fa.status_string(st)} {word:#x}")

    copies = 1 if args.l2_warm else rotation_copies(w.algorithmic_bytes, args.steps)
    if copies == 1 and not args.l2_warm:
        # --- device-timed region: K launches, per-launch events on the launch stream
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        t_begin = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        sync_all()
        with ClockSampler(local) as clocks:
            with torch.cuda.stream(stream):
                t_begin.record(stream)
                for i in range(args.steps):
                    starts[i].record(stream)
                    step()
                    ends[i].record(stream)
                t_end.record(stream)
            sync_all()
        clock_summary = clocks.summary()
        total_ms = t_begin.elapsed_time(t_end)
        launch_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
        total_ms = max_over_ranks(total_ms, dev)
        avg_launch_ms = max_over_ranks(sum(launch_ms) / len(launch_ms), dev)
    else:
        # --- a workload smaller than L2: the K launches cycle through copies of
        # the buffers and run from one CUDA graph (eager launches of a few
        # microseconds would time the host); per launch = total / K.
        bufs = [(qd, kd, vd, od, lsed)] + [
            (qd.clone(), kd.clone(), vd.clone(), torch.empty_like(od), torch.empty_like(lsed))
            for _ in range(copies - 1)]

        def launch(i):
            a = bufs[i % copies]
            fa.fa_fwd(a[0], a[1], a[2], causal=w.causal, scale=w.scale, out=a[3], lse=a[4],
                      stream=stream, schedule=sched)

        total_ms, clock_summary = time_graph(launch, args.steps, 1, stream, local, sync_all,
                                             flush_l2=not args.l2_warm)
        total_ms = max_over_ranks(total_ms, dev)
        avg_launch_ms = total_ms / args.steps
    st, word = fa.device_status(stream.cuda_stream)
    if st != fa.FA_OK:
        raise SystemExit(f"kernel status {fa.status_string(st)} {word:#x}")

    flops_step = w.flops
    ms_per_step = total_ms / args.steps
    value = world * flops_step * args.steps / (total_ms / 1e3) / 1e12

    # --- end to end through the C ABI with host buffers (fa_fwd_host): every
    # step copies Q, K, V from pinned host memory, runs the forward and copies
    # O and LSE back, the transfers of chunks of heads overlapped with the
    # attention of others.
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    oh = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    lh = torch.empty((w.B, w.H, w.N), dtype=torch.float32).pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = oh.numel() * oh.element_size() + lh.numel() * lh.element_size()
    e2e_ws = torch.empty(fa.host_workspace_bytes(w.B, w.H, w.N, w.d), dtype=torch.uint8,
                         device=dev)

    def e2e_step():
        fa.fa_fwd_host(qh, kh, vh, causal=w.causal, scale=w.scale, out=oh, lse=lh,
                       workspace=e2e_ws, stream=stream, device=dev)

    with torch.cuda.stream(stream):
        e2e_step()
    sync_all()
    e_begin = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e_begin.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e_end.record(stream)
    sync_all()
    e2e_ms = max_over_ranks(e_begin.elapsed_time(e_end), dev)
    e2e_value = world * flops_step * e2e_steps / (e2e_ms / 1e3) / 1e12

    peak, peak_sustained, peak_src = load_peaks()
    achieved = flops_step / (avg_launch_ms / 1e3) / 1e12
    traffic = load_traffic(w.name)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w, world, sched, copies, args.l2_warm),
        "pct_of_peak": 100.0 * value / world / peak,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{peak_src} bf16_tflops (burst)",
                     "frac_of_sustained": (achieved / peak_sustained) if peak_sustained else None,
                     "frac_of_nominal": achieved / NOMINAL_BF16_TFLOPS,
                     "kernel": fwd_kernel_name(w.d), "avg_launch_ms": avg_launch_ms},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps, "entry": "fa_fwd_host",
                "ms_per_step": e2e_ms / e2e_steps},
        "gpu_launches": args.steps,
        "clocks": clock_summary,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, secs, desc = time_oracle_sample(w, q, k, v, target_s=args.cpu_seconds)
        line["cpu_baseline"] = {"value": tf, "unit": UNIT, "cores": blas_threads() or os.cpu_count(),
                                "kind": "oracle", "sample": desc, "seconds": secs}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_decode(args):
    import torch

    import exact_attention_122_b200 as fa

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    w = synth.DECODE_WORKLOAD
    if args.decode_batch != w.B:
        # a smaller batch of the same shape (profiling captures); traffic
        # and time scale with the batch
        w = synth.DecodeWorkload(f"{w.name}_b{args.decode_batch}", args.decode_batch, w.H, w.Nq,
                                 w.Nk, w.d, w.causal, w.seed)
    q, k, v = (t.to(dev) for t in synth.draw_decode_qkv(w.B, w.H, w.Nq, w.Nk, w.d, w.seed))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
    ws = torch.empty(fa.decode_workspace_bytes(w.B, w.H, w.Nq, w.Nk, w.d), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step():
        fa.fa_fwd_decode(q, k, v, causal=w.causal, out=o, lse=lse, workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clocks:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(args.steps):
                step()
            e1.record(stream)
        torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / args.steps
    gbs = w.algorithmic_bytes / (ms / 1e3) / 1e9
    try:
        with open(PEAKS_FILE) as f:
            peak, src = float(json.load(f)["hbm_gbs"]), "measured hbm_gbs"
    except (OSError, KeyError, ValueError):
        peak, src = 6650.0, "fallback"
    line = {"metric": "decode attention effective HBM GB/s (1 GPU)", "value": gbs, "unit": "GB/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "Nq": w.Nq, "Nk": w.Nk, "d": w.d,
                       "causal": w.causal,
                       "l2": f"K+V {w.kv_bytes / 1e9:.1f} GB > 126 MB L2; no flush"},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                         "frac": gbs / peak, "traffic": load_traffic(w.name, DECODE_KERNEL_SOURCE),
                         "traffic_kernel": "decode_mma_kernel", "peak_source": src,
                         "kernel": "decode_mma_kernel + decode_merge_kernel"},
            "gpu_launches": 2 * args.steps, "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)
    return 0


def run_bwd(args):
    """Backward pass of the headline workload: one step = fa_bwd (D pre-pass,
    the main gradient kernel, dQ conversion) on inputs and forward outputs
    already in device memory.  FLOPs: the five matrix products of the
    recomputing backward (S, dP, dV, dK, dQ), 2.5x the forward's count."""
    import torch

    import exact_attention_122_b200 as fa

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    w = synth.workload(args.workload)
    elems = w.B * w.H * w.N * w.d
    step_bytes = 8 * 2 * elems + 4 * w.B * w.H * w.N    # Q,K,V,O,dO in, dQ,dK,dV out; LSE
    require_beyond_l2(step_bytes, args.steps, "--bwd")
    q, k, v = (t.to(dev) for t in synth.workload_qkv(w))
    dout = synth.draw_dout(w.B, w.H, w.N, w.d, seed=w.seed).to(dev)
    stream = torch.cuda.Stream(device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.bwd_workspace_bytes(w.B, w.H, w.N, w.d), dtype=torch.uint8, device=dev)
    with torch.cuda.stream(stream):
        fa.fa_fwd(q, k, v, causal=w.causal, out=o, lse=lse, stream=stream)

    def step():
        fa.fa_bwd(q, k, v, o, lse, dout, causal=w.causal, dq=dq, dk=dk, dv=dv, workspace=ws,
                  stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clocks:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(args.steps):
                step()
            e1.record(stream)
        torch.cuda.synchronize(dev)
    st, word = fa.device_status(stream.cuda_stream)
    if st != fa.FA_OK:
        raise SystemExit(f"kernel status {fa.status_string(st)} {word:#x}")
    ms = e0.elapsed_time(e1) / args.steps
    flops = 2.5 * w.flops
    value = flops / (ms / 1e3) / 1e12
    peak, peak_sus, peak_src = load_peaks()
    line = {"metric": "attention backward TFLOP/s (1 GPU)", "value": value, "unit": "TFLOP/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                       "causal": w.causal, "flops_per_step": flops,
                       "l2": l2_note(step_bytes, 1)},
            "roofline": {"bound": "tensor", "achieved": value, "peak": peak, "unit": "TFLOP/s",
                         "frac": value / peak,
                         "traffic": load_traffic(w.name + "_bwd", BWD_KERNEL_SOURCE),
                         "traffic_kernel": "bwd_kernel_x", "peak_source": peak_src,
                         "kernel": "bwd_prep + bwd_kernel_x + bwd_dq_out (whole step)"},
            "gpu_launches": 3 * args.steps, "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)
    return 0


def run_fp8(args):
    """FP8 forward of the workload's shape: one step = fa_fwd_fp8 (V^T pass and
    the attention kernel) on E4M3 inputs already in device memory."""
    import torch

    import exact_attention_122_b200 as fa

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    w = synth.workload(args.workload)
    step_bytes = 5 * w.B * w.H * w.N * w.d + 4 * w.B * w.H * w.N   # E4M3 Q,K,V in, bf16 O out; LSE
    require_beyond_l2(step_bytes, args.steps, "--fp8")
    (q8, k8, v8), (sq, sk, sv) = synth.draw_qkv_fp8(w.B, w.H, w.N, w.d, seed=w.seed,
                                                     qk_std=w.qk_std)
    q8, k8, v8 = q8.to(dev), k8.to(dev), v8.to(dev)
    stream = torch.cuda.Stream(device=dev)
    o = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    ws = torch.empty(fa.fp8_workspace_bytes(w.B, w.H, w.N, w.d), dtype=torch.uint8, device=dev)

    def step():
        fa.fa_fwd_fp8(q8, k8, v8, sq, sk, sv, causal=w.causal, out=o, lse=lse, workspace=ws,
                      stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clocks:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(args.steps):
                step()
            e1.record(stream)
        torch.cuda.synchronize(dev)
    st, word = fa.device_status(stream.cuda_stream)
    if st != fa.FA_OK:
        raise SystemExit(f"kernel status {fa.status_string(st)} {word:#x}")
    ms = e0.elapsed_time(e1) / args.steps
    value = w.flops / (ms / 1e3) / 1e12
    peak_bf16, _, peak_src = load_peaks()
    # FP8 dense peak: the measured bf16 peak times the nominal FP8 / bf16 ratio (4.5 / 2.25).
    peak = 2.0 * peak_bf16
    line = {"metric": "attention fwd TFLOP/s, FP8 E4M3 inputs (1 GPU)", "value": value,
            "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "dtype": "e4m3", "data": "synthetic",
            "config": {"workload": w.name + "_fp8", "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                       "causal": w.causal, "l2": l2_note(step_bytes, 1)},
            "roofline": {"bound": "tensor", "achieved": value, "peak": peak, "unit": "TFLOP/s",
                         "frac": value / peak, "traffic": load_traffic(w.name + "_fp8"),
                         "traffic_kernel": "fa_fwd_kernel<128, 8, true>",
                         "peak_source": f"{peak_src} bf16 x 2 (nominal FP8/bf16 ratio)",
                         "kernel": "transpose_v_e4m3 + fa_fwd_kernel<128, 8, true> (whole step)"},
            "gpu_launches": 3 * args.steps, "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)
    return 0


def run_sweep(args):
    import torch

    import exact_attention_122_b200 as fa

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.Stream(device=dev)
    peak, _, peak_src = load_peaks()

    def sync_all():
        torch.cuda.synchronize(dev)

    for N in synth.SWEEP_SEQ_LENS:
        w = synth.sweep_workload(N)
        sched = bench_schedule(args.schedule, w, torch.cuda.get_device_properties(dev).multi_processor_count)
        q, k, v = (t.to(dev) for t in synth.workload_qkv(w))
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
        # at least ~200 ms of timed work per length, and at least args.steps launches
        steps = max(args.steps, int(0.2 / max(w.flops / 1.0e15, 1e-6)))
        copies = rotation_copies(w.algorithmic_bytes, steps)
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                fa.fa_fwd(q, k, v, causal=True, out=o, lse=lse, stream=stream,
                          schedule=sched)
        sync_all()
        if copies == 1:
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            with ClockSampler(0) as clocks:
                with torch.cuda.stream(stream):
                    e0.record(stream)
                    for _ in range(steps):
                        fa.fa_fwd(q, k, v, causal=True, out=o, lse=lse, stream=stream,
                                  schedule=sched)
                    e1.record(stream)
                sync_all()
            total_ms, clock_summary = e0.elapsed_time(e1), clocks.summary()
        else:
            # One graph of G launches (a multiple of the copy count, so the
            # rotation runs on across replays), replayed until >= steps.
            bufs = [(q, k, v, o, lse)] + [
                (q.clone(), k.clone(), v.clone(), torch.empty_like(o), torch.empty_like(lse))
                for _ in range(copies - 1)]
            G = copies * math.ceil(min(steps, 512) / copies)
            R = math.ceil(steps / G)
            steps = G * R

            def launch(i):
                a = bufs[i % copies]
                fa.fa_fwd(a[0], a[1], a[2], causal=True, out=a[3], lse=a[4], stream=stream,
                          schedule=sched)

            total_ms, clock_summary = time_graph(launch, G, R, stream, 0, sync_all)
            del bufs
        ms = total_ms / steps
        st, word = fa.device_status(stream.cuda_stream)
        if st != fa.FA_OK:
            raise SystemExit(f"kernel status {fa.status_string(st)} {word:#x}")
        value = w.flops / (ms / 1e3) / 1e12
        print(json.dumps({"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
                          "steps": steps, "warmup": args.warmup, "ms_per_step": ms,
                          "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
                          "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                                     "causal": True, "schedule": sched,
                                     "l2": l2_note(w.algorithmic_bytes, copies)},
                          "pct_of_peak": 100.0 * value / peak, "peak_source": peak_src,
                          "gpu_launches": steps, "clocks": clock_summary}),
              flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=WORKLOAD_INDEX,
                    help="workload index (1..5); the default is the headline workload")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target length of the oracle CPU-baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--schedule", choices=["auto", "static", "dynamic"], default="auto",
                    help="work distribution: fa_fwd_dynamic, fa_fwd (static), or auto (default: "
                         "dynamic from 4 to 12 units of 256 rows per SM, static otherwise)")
    ap.add_argument("--l2-warm", action="store_true",
                    help="time the forward line on one reused set of buffers without an L2 flush "
                         "(graph-replayed): the L2-warm figure for workloads that fit in L2")
    ap.add_argument("--decode", action="store_true",
                    help="time the decode-shaped path (HBM-bound) instead of the headline line")
    ap.add_argument("--decode-batch", type=int, default=synth.DECODE_WORKLOAD.B,
                    help="batch of the --decode line (default: the decode workload's); smaller "
                         "batches keep profiling captures to a few GB")
    ap.add_argument("--fp8", action="store_true",
                    help="time the FP8 (E4M3) forward of the workload's shape")
    ap.add_argument("--bwd", action="store_true",
                    help="time the backward pass (fa_bwd) of the workload instead of the forward")
    ap.add_argument("--sweep", action="store_true",
                    help="print the sequence-length sweep curve instead of the headline line")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.steps < 1:
        raise SystemExit("--steps must be >= 1")
    if args.sweep:
        return run_sweep(args)
    if args.bwd:
        return run_bwd(args)
    if args.fp8:
        return run_fp8(args)
    if args.decode:
        return run_decode(args)
    w = synth.workload(args.workload)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
