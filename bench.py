"""Benchmark of the exact attention forward on B200.

Default workload: the full long-context causal forward (B=1, Hq=Hkv=32,
N=131072, d=128), the largest of the single-GPU workloads, bf16 inputs resident
in HBM.  One step = one forward over the whole batch (one kernel launch).
Metric: TFLOP/s counting 4*d FLOPs per visible (query, key) pair.  Inputs
(3 GiB of q, k, v) are larger than the 126 MB L2, so no flush is needed between
steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload dense|gqa|swa|long|tiny|decode_*] [--no-cpu-baseline]
                  [--pass fwd|bwd|decode|ring] [--dtype bf16|fp8]

``--pass bwd`` times the backward pass instead (one GPU; 10*d FLOPs per visible
pair, the five products of the gradient).  ``--pass decode`` times one decoding
step against a paged KV cache (``--workload decode_gqa|decode_mha|decode_swa|
decode_spec``; one GPU; GB/s of algorithmic bytes against the measured HBM
bandwidth).  ``--dtype fp8`` runs the forward on E4M3 inputs (peak: the measured bf16
figure x 2).  ``--pass ring`` runs ring attention with all its ranks emulated on one GPU
(``--ring-ranks R``).

With --gpus N > 1 the script runs under torchrun, one rank per GPU, and rank 0
prints one JSON line with the max-over-ranks time.  By default every rank runs
its own shard of the global batch (weak scaling, no data-path collective);
``--split heads`` instead splits the one workload's (batch, KV-group) units
into contiguous ranges, one per rank (strong scaling, still no collective:
``exact_io_aware_72_b200.shard``).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from harness.inputs import DECODE_WORKLOADS, WORKLOADS, make_qkv, sample_rows  # noqa: E402

METRIC = "attention fwd TFLOP/s (bf16, causal/window-adjusted) and % of B200 dense peak"
FP8_METRIC = "attention fwd TFLOP/s (E4M3 inputs, causal/window-adjusted) and % of B200 dense fp8 peak"
FP8_OVER_BF16 = 2.0  # nominal dense fp8 / bf16 tensor rate (4.5 / 2.25 PFLOP/s)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ["exact_io_aware_72_b200/csrc/attn_fwd.cu", "exact_io_aware_72_b200/csrc/attn_fwd_kernel.cuh",
                  "exact_io_aware_72_b200/csrc/sm100_ptx.cuh"]
# DRAM bytes per launch of the forward kernel from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum), keyed by the hash of the kernel
# sources it was taken on; reported only while the sources still match.  The
# long workload's figure is the capture of the same kernel on a causal
# N = 32768 case (1, 32, 32, 32768, 128) times 4: DRAM bytes grow linearly in N.
# The FP8 long figure is a capture of the full launch (E4M3 q, k, v: 1.2 GiB).
NCU_TRAFFIC = {
    ("dense", "e2664b285cb35e2b"): 410178304 + 111494656,
    ("long", "e2664b285cb35e2b"): 4 * (937351680 + 253613312),
    ("long_fp8", "e2664b285cb35e2b"): 2079931136 + 1068808704,
}


def visible_pairs(N: int, mask: str, window) -> int:
    """Visible (query, key) pairs of one head: N^2, N(N+1)/2, or N w - w(w-1)/2."""
    if mask == "full":
        return N * N
    if mask == "causal" or (mask == "sliding_window" and window >= N):
        return N * (N + 1) // 2
    w = window
    return N * w - w * (w - 1) // 2


def workload_flops(w, batch: int) -> int:
    return 4 * batch * w.Hq * w.d * visible_pairs(w.N, w.mask, w.window)


def kernel_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


DECODE_KERNEL_SOURCES = ["exact_io_aware_72_b200/csrc/attn_decode_kernel.cuh", "exact_io_aware_72_b200/csrc/sm100_ptx.cuh"]
# DRAM bytes per launch of the decoding kernel from one ncu capture, keyed by
# workload and the hash of the decoding kernel's device sources.
DECODE_NCU_TRAFFIC = {
    ("decode_gqa", "786921213997f59a"): 537017856 + 3168000,
}


def decode_kernel_hash() -> str:
    h = hashlib.sha256()
    for rel in DECODE_KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons while it runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.marks = [None, None]

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu=timestamp,{self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, i):
        self.marks[i] = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        t0, t1 = self.marks
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, line in self.lines:
            if t0 is not None and not (t0 - 0.05 <= ts <= t1 + 0.15):
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- distributed
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (a timing reduction, not data)."""
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ----------------------------------------------------------------- oracle (CPU)
def oracle_sample(w, q, k, v, rows, heads, scale):
    """Time the fp64 oracle on `rows` of `heads` (list of (b, h)); returns
    (seconds, visible-pair FLOPs done, threads)."""
    import oracle
    from threadpoolctl import threadpool_info
    g = w.Hq // w.Hkv
    # host copies prepared outside the timed region
    work = []
    for b, h in heads:
        work.append((q[b:b + 1, h:h + 1].float().cpu().numpy(), k[b:b + 1, h // g:h // g + 1].float().cpu().numpy(),
                     v[b:b + 1, h // g:h // g + 1].float().cpu().numpy()))
    t0 = time.perf_counter()
    for qh, kh, vh in work:
        oracle.attention(qh, kh, vh, scale, w.mask_kind, w.window, rows=rows)
    dt = time.perf_counter() - t0
    counts = oracle.visible_count_per_row(w.N, w.mask_kind, w.window)[rows]
    flops = 4 * w.d * int(counts.sum()) * len(heads)
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return dt, flops, threads


def cpu_baseline(w, q, k, v, target_s=15.0):
    """Oracle on host cores on a bounded sample of the workload (about target_s
    seconds): seeded query rows of as many heads as fit, all heads if they fit."""
    rows = sample_rows(w.N, w.window, w.seed + 100, count=min(w.N, 256))
    dt, _, _ = oracle_sample(w, q, k, v, rows, [(0, 0)], w.scale)
    n_heads = max(1, min(w.B * w.Hq, int(target_s / max(dt, 1e-3))))
    if n_heads == w.B * w.Hq and dt * n_heads < target_s / 2 and len(rows) < w.N:
        rows = sample_rows(w.N, w.window, w.seed + 100,
                           count=min(w.N, int(len(rows) * target_s / max(dt * n_heads, 1e-3) / 2)))
    heads = [(i // w.Hq, i % w.Hq) for i in range(n_heads)]
    dt, flops, threads = oracle_sample(w, q, k, v, rows, heads, w.scale)
    # The same oracle on one thread, on a smaller sample (one head, up to 64 rows).
    from threadpoolctl import threadpool_limits
    rows1 = rows[:: max(1, len(rows) // 64)][:64]
    with threadpool_limits(limits=1):
        dt1, flops1, _ = oracle_sample(w, q, k, v, rows1, heads[:1], w.scale)
    pairs = flops // (4 * w.d)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "rows_per_s": len(rows) * n_heads / dt, "pairs_per_s": pairs / dt,
            "one_thread": {"value": flops1 / dt1 / 1e12, "unit": "TFLOP/s", "rows_per_s": len(rows1) / dt1,
                           "pairs_per_s": flops1 // (4 * w.d) / dt1},
            "sample": f"{len(rows)} seeded query rows x {n_heads} heads of the {w.name} workload "
                      f"(fp64 NumPy, scores materialised), {dt:.1f} s; one thread: {len(rows1)} rows of "
                      f"one head, {dt1:.2f} s",
            "seconds": dt}


def fp8_cpu_baseline(w, q8, k8, v8, sq, sk, sv):
    """The fp64 FP8 oracle (decode, dequantise, forward definition) on 256
    seeded query rows of one head, on the host cores."""
    from threadpoolctl import threadpool_info
    from oracle import attention_fp8 as O8
    rows = sample_rows(w.N, w.window, w.seed + 100, count=min(w.N, 256))
    g = w.Hq // w.Hkv
    qh, kh, vh = (t[:1, :1].cpu().numpy() for t in (q8, k8[:, :1], v8[:, :1]))
    t0 = time.perf_counter()
    O8.attention_fp8(qh, kh, vh, sq, sk, sv, w.scale, w.mask_kind, w.window, rows=rows)
    dt = time.perf_counter() - t0
    from oracle import visible_count_per_row
    flops = 4 * w.d * int(visible_count_per_row(w.N, w.mask_kind, w.window)[rows].sum())
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{len(rows)} seeded query rows of one head of the {w.name} workload (E4M3 decoded, "
                      f"fp64 NumPy, scores materialised), {dt:.1f} s; group size {g}"}


# ----------------------------------------------------------------- arms
def run_reference(args, w):
    """The oracle as the reference arm: each step is a bounded sample of the
    workload (64 seeded rows of a few heads) on the host cores."""
    world, rank, _ = dist_env()
    if rank != 0:
        return
    q, k, v = make_qkv(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed, device="cpu", sharp=w.sharp)
    rows = sample_rows(w.N, w.window, w.seed + 100, count=64)
    heads = [(0, h) for h in range(min(4, w.Hq))]
    for _ in range(args.warmup):
        oracle_sample(w, q, k, v, rows, heads[:1], w.scale)
    total_s, total_f, threads = 0.0, 0, 1
    for _ in range(args.steps):
        dt, fl, threads = oracle_sample(w, q, k, v, rows, heads, w.scale)
        total_s += dt
        total_f += fl
    value = total_f / total_s / 1e12
    rows_per_s = len(rows) * len(heads) * args.steps / total_s
    pairs_per_s = total_f / (4 * w.d) / total_s
    sample = f"{len(rows)} seeded query rows x {len(heads)} heads of the {w.name} workload per step (fp64 NumPy)"
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1000 * total_s / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d,
                       "mask": w.mask, "window": w.window, "global_batch": w.B, "seq_len": w.N,
                       "parallelism": "cpu"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "rows_per_s": rows_per_s, "pairs_per_s": pairs_per_s, "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, w):
    world, rank, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    from exact_io_aware_72_b200 import fwd, fwd_fp8, fwd_fp8_host, fwd_host
    fp8 = args.dtype == "fp8"

    split_heads = args.split == "heads" and world > 1
    # Each rank runs its own shard of the global batch: B sequences seeded by rank;
    # or (--split heads) its contiguous range of the one workload's (b, KV-group) units.
    seed = w.seed if split_heads else w.seed + 1000 * rank
    if fp8:
        from harness.inputs import make_qkv_fp8
        (q, sq), (k, sk), (v, sv) = make_qkv_fp8(w.B, w.Hq, w.Hkv, w.N, w.d, seed, device=device, sharp=w.sharp)
    else:
        q, k, v = make_qkv(w.B, w.Hq, w.Hkv, w.N, w.d, seed, device=device, sharp=w.sharp)
    total_flops = workload_flops(w, w.B) * (1 if split_heads else world)
    flops = workload_flops(w, w.B)   # this rank's work per step
    units = None
    if split_heads:
        from exact_io_aware_72_b200 import shard
        q, k, v, (u0, u1) = shard.head_shard(q, k, v, world, rank)
        units = shard.shard_sizes(w.B, w.Hkv, world)
        if q is None:
            raise SystemExit(f"--split heads: rank {rank} has no (batch, KV-group) unit; use fewer GPUs")
        flops = workload_flops(w, w.B) * (u1 - u0) // (w.B * w.Hkv)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=device)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        if fp8:
            fwd_fp8(q, k, v, sq, sk, sv, scale=w.scale, mask=w.mask, window=w.window, out=out, lse=lse,
                    stream=stream)
        else:
            fwd(q, k, v, scale=w.scale, mask=w.mask, window=w.window, out=out, lse=lse, stream=stream)

    clocks = ClockSampler(local)
    if rank == 0:
        clocks.start()
        time.sleep(0.3)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    barrier(world, device)
    torch.cuda.synchronize(device)
    clocks.mark(0)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    evs[0].record(stream)
    for i in range(args.steps):
        step()
        evs[i + 1].record(stream)
    torch.cuda.synchronize(device)
    clocks.mark(1)
    barrier(world, device)
    per_launch_ms = [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)]
    total_ms = evs[0].elapsed_time(evs[-1])
    total_ms = max_over_ranks(total_ms, world, device)
    clk = clocks.stop() if rank == 0 else None

    # End to end through the public host-buffer call: pinned q, k, v in, out and lse back.
    # The pinned host outputs and the device staging buffers are the caller's and are
    # set up once, as a serving loop would; every step copies all of q, k, v up and
    # all of out, lse down.
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    hout = torch.empty(out.shape, dtype=torch.bfloat16, pin_memory=True)
    hlse = torch.empty(lse.shape, dtype=torch.float32, pin_memory=True)
    staging = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(out),
               torch.empty_like(lse))

    # The library cuts the job into chunks of (batch, key/value head) units and
    # overlaps each chunk's upload, kernel and download on three streams.
    def e2e_step():
        if fp8:
            fwd_fp8_host(hq, hk, hv, sq, sk, sv, device=device, scale=w.scale, mask=w.mask, window=w.window,
                         out=hout, lse=hlse, staging=staging)
        else:
            fwd_host(hq, hk, hv, device=device, scale=w.scale, mask=w.mask, window=w.window, out=hout, lse=hlse,
                     staging=staging)

    for _ in range(2):
        e2e_step()
    e2e_steps = max(3, min(args.steps, 20))
    torch.cuda.synchronize(device)
    barrier(world, device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, device)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    d2h = out.numel() * out.element_size() + lse.numel() * lse.element_size()

    if rank == 0:
        peaks, peak_src = load_peaks()
        avg_launch_s = statistics.mean(per_launch_ms) / 1e3
        achieved = flops / avg_launch_s / 1e12
        peak = float(peaks["bf16_tflops"]) * (FP8_OVER_BF16 if fp8 else 1.0)
        value = total_flops * args.steps / (total_ms / 1e3) / 1e12
        traffic = NCU_TRAFFIC.get((w.name + ("_fp8" if fp8 else ""), kernel_hash()))
        line = {
            "metric": FP8_METRIC if fp8 else METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "strong" if split_heads else "weak", "vs_baseline": None,
            "dtype": "e4m3" if fp8 else "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d,
                       "mask": w.mask, "window": w.window, "sharp_rows": w.sharp,
                       "global_batch": w.B if split_heads else w.B * world, "seq_len": w.N,
                       "parallelism": f"heads{world}" if split_heads else f"dp{world}",
                       "l2": "inputs larger than L2 (no flush)"},
            "frac_of_peak": value / world / peak,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": (f"{peak_src} bf16_tflops (burst) x {FP8_OVER_BF16} (nominal fp8/bf16)"
                                         if fp8 else f"{peak_src} bf16_tflops (burst)"),
                         "frac_of_sustained": achieved / (float(peaks.get("bf16_tflops_sustained", peak)) *
                                                          (FP8_OVER_BF16 if fp8 else 1.0))},
            "gpu_launches": args.steps,
            "launch_ms": {"median": statistics.median(per_launch_ms), "best": min(per_launch_ms)},
            "clocks": clk,
            "e2e": {"value": total_flops * e2e_steps / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "path": ("attn_fwd_fp8_host" if fp8 else "attn_fwd_host") + " from pinned host memory, "
                            "8 chunks, copies overlapped with the kernels",
                    "ms_per_step": e2e_ms / e2e_steps},
        }
        if units is not None:
            line["config"]["units_per_rank"] = units
        if not args.no_cpu_baseline and world == 1:   # the host-core baseline is an N = 1 figure
            if fp8:
                line["cpu_baseline"] = fp8_cpu_baseline(w, q, k, v, sq, sk, sv)
            else:
                line["cpu_baseline"] = cpu_baseline(w, q, k, v, target_s=args.cpu_seconds)
                line["cpu_baseline"].pop("seconds", None)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


BWD_METRIC = "attention bwd TFLOP/s (bf16, 10*d FLOPs per visible pair) and % of B200 dense peak"


def bwd_cpu_baseline(w, q, k, v, do, target_s=15.0):
    """The fp64 backward oracle on host cores for one query head (with its KV
    head) over a prefix of the sequence short enough to finish in seconds."""
    import oracle.attention_bwd_fp64 as G
    from oracle import attention_fp64 as F
    n = min(w.N, 2048)
    while True:
        qs = q[:1, :1, :n].float().numpy()
        ks = k[:1, :1, :n].float().numpy()
        vs = v[:1, :1, :n].float().numpy()
        ds = do[:1, :1, :n].float().numpy()
        t0 = time.perf_counter()
        G.attention_bwd(qs, ks, vs, ds, w.scale, F.MASK_CAUSAL if w.mask == "causal" else
                        (F.MASK_FULL if w.mask == "full" else F.MASK_SLIDING_WINDOW), w.window)
        dt = time.perf_counter() - t0
        if dt > target_s / 8 or n >= min(w.N, 8192):
            break
        n = min(w.N, 8192, n * 2)
    flops = 10 * w.d * visible_pairs(n, w.mask, w.window)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
            "sample": f"one query head and its KV head, first {n} positions of the {w.name} workload "
                      f"(fp64 NumPy, scores materialised), {dt:.1f} s"}


def run_backward(args, w):
    """Backward pass on one GPU: each step is one attn_bwd call on the forward's
    out and lse and a seeded dO (three kernels: D, then for d = 128 the fused
    key-tile kernel and the dQ conversion after zeroing the fp32 dQ sums, for
    d = 64 the dQ and dK/dV kernels)."""
    from harness.inputs import make_dout
    from exact_io_aware_72_b200 import bwd, fwd
    from exact_io_aware_72_b200.attn import load_library
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    q, k, v = make_qkv(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed, device=device, sharp=w.sharp)
    do = make_dout(w.B, w.Hq, w.N, w.d, w.seed, device=device)
    out, lse = fwd(q, k, v, scale=w.scale, mask=w.mask, window=w.window)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    det = bool(args.bwd_deterministic)
    fused = w.d == 128 and w.Hq == w.Hkv and not det
    ws_bytes = int(load_library().attn_bwd_workspace_bytes(w.B, w.Hq, w.N)) if fused else 4 * w.B * w.Hq * w.N
    ws = torch.empty(ws_bytes // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        bwd(q, k, v, out, lse, do, scale=w.scale, mask=w.mask, window=w.window, dq=dq, dk=dk, dv=dv,
            workspace=ws, stream=stream, deterministic=det)

    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    clocks.mark(0)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    evs[0].record(stream)
    for i in range(args.steps):
        step()
        evs[i + 1].record(stream)
    torch.cuda.synchronize(device)
    clocks.mark(1)
    per_launch_ms = [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)]
    total_ms = evs[0].elapsed_time(evs[-1])
    clk = clocks.stop()
    flops = 10 * w.B * w.Hq * w.d * visible_pairs(w.N, w.mask, w.window)
    peaks, peak_src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    achieved = flops / (statistics.mean(per_launch_ms) / 1e3) / 1e12
    line = {
        "metric": BWD_METRIC, "pass": "bwd", "value": flops * args.steps / (total_ms / 1e3) / 1e12,
        "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d, "mask": w.mask,
                   "window": w.window, "sharp_rows": w.sharp, "l2": "inputs larger than L2 (no flush)",
                   "bwd_path": "fused key-tile kernel" if fused else "dQ kernel + dK/dV kernel"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "traffic": None, "peak_source": f"{peak_src} bf16_tflops (burst)",
                     "frac_of_sustained": achieved / float(peaks.get("bf16_tflops_sustained", peak))},
        "gpu_launches": 3 * args.steps,
        "launch_ms": {"median": statistics.median(per_launch_ms), "best": min(per_launch_ms)},
        "clocks": clk,
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = bwd_cpu_baseline(w, q.cpu(), k.cpu(), v.cpu(), do.cpu(), args.cpu_seconds)
    print(json.dumps(line), flush=True)


DEC_METRIC = "attention decode GB/s (bf16 paged KV cache, algorithmic bytes) and % of measured HBM bandwidth"


def decode_bytes(w, lens) -> int:
    """Algorithmic bytes of one decoding step: K and V (bf16) of every position
    a step's queries can see (from max(0, L - Nq - window + 1) under a window,
    else from 0, to L - 1) for each KV head, plus q and out (bf16) and lse."""
    keys = 0
    for L in (int(x) for x in lens):
        lo = max(0, L - w.Nq - w.window + 1) if w.mask == "sliding_window" else 0
        keys += L - lo
    return 2 * 2 * w.d * w.Hkv * keys + w.B * w.Hq * w.Nq * (2 * 2 * w.d + 4)


def decode_cpu_sample(w, inp, seqs):
    """The fp64 decoding oracle on the sequences ``seqs`` (host copies made
    outside the timed region); returns (seconds, algorithmic bytes, threads)."""
    from threadpoolctl import threadpool_info
    from dataclasses import replace
    from oracle import attention_decode_fp64 as DO
    table = inp["block_table"].cpu().numpy()
    lens = inp["seq_lens"].cpu().numpy()
    used = sorted({int(pg) for b in seqs for pg in table[b] if pg >= 0})
    remap = {pg: i for i, pg in enumerate(used)}
    idx = torch.as_tensor(used, dtype=torch.long, device=inp["k_cache"].device)
    kc = inp["k_cache"].index_select(0, idx).float().cpu().numpy()
    vc = inp["v_cache"].index_select(0, idx).float().cpu().numpy()
    sub = np.array([[remap.get(int(pg), -1) for pg in table[b]] for b in seqs], dtype=np.int64)
    q = inp["q"][list(seqs)].float().cpu().numpy()
    t0 = time.perf_counter()
    DO.decode_attention(q, kc, vc, sub, lens[list(seqs)], w.scale, w.mask_kind, w.window)
    dt = time.perf_counter() - t0
    nbytes = decode_bytes(replace(w, B=len(seqs)), lens[list(seqs)])
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return dt, nbytes, threads


def run_decode(args, w):
    """Decoding step on one GPU: each step is one attn_decode call (the
    decoding kernel, plus the split merge when the step uses splits) over the
    workload's paged KV cache, resident in HBM."""
    from harness.inputs import make_decode_workload
    from exact_io_aware_72_b200 import decode, decode_num_splits, decode_workspace_bytes
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    inp = make_decode_workload(w, device=device)
    lens = inp["seq_lens"].cpu().numpy()
    max_len = int(lens.max())
    splits = args.splits or decode_num_splits(w.B, w.Hq, w.Hkv, w.Nq, max_len, w.mask, w.window)
    out = torch.empty_like(inp["q"])
    lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=device)
    ws_bytes = decode_workspace_bytes(w.B, w.Hq, w.Nq, w.d, splits)
    ws = torch.zeros(ws_bytes // 4, dtype=torch.float32, device=device)  # counter must start at zero
    stream = torch.cuda.current_stream(device)
    nbytes = decode_bytes(w, lens)

    def step(q=inp["q"], bt=inp["block_table"], sl=inp["seq_lens"]):
        decode(q, inp["k_cache"], inp["v_cache"], bt, sl, scale=w.scale, mask=w.mask, window=w.window,
               num_splits=splits, out=out, lse=lse, workspace=ws, stream=stream)

    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    clocks.mark(0)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    evs[0].record(stream)
    for i in range(args.steps):
        step()
        evs[i + 1].record(stream)
    torch.cuda.synchronize(device)
    clocks.mark(1)
    per_step_ms = [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)]
    total_ms = evs[0].elapsed_time(evs[-1])
    clk = clocks.stop()

    # End to end: the step's new inputs (q, page table, lengths) from pinned host
    # memory, the result (out, lse) back; the KV cache stays resident in HBM.
    hq, hbt, hsl = (t.cpu().pin_memory() for t in (inp["q"], inp["block_table"], inp["seq_lens"]))
    ho = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    hl = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    dq, dbt, dsl = torch.empty_like(inp["q"]), torch.empty_like(inp["block_table"]), torch.empty_like(inp["seq_lens"])

    def e2e_step():
        dq.copy_(hq, non_blocking=True)
        dbt.copy_(hbt, non_blocking=True)
        dsl.copy_(hsl, non_blocking=True)
        step(dq, dbt, dsl)
        ho.copy_(out, non_blocking=True)
        hl.copy_(lse, non_blocking=True)

    for _ in range(2):
        e2e_step()
    e2e_steps = max(3, min(args.steps, 20))
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = e0.elapsed_time(e1)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hbt, hsl))
    d2h = ho.numel() * ho.element_size() + hl.numel() * hl.element_size()

    peaks, peak_src = load_peaks()
    peak = float(peaks["hbm_gbs"])
    achieved = nbytes / (statistics.mean(per_step_ms) / 1e3) / 1e9
    line = {
        "metric": DEC_METRIC, "pass": "decode", "value": nbytes * args.steps / (total_ms / 1e3) / 1e9,
        "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Nq": w.Nq, "d": w.d,
                   "seq_len_min": int(lens.min()), "seq_len_max": max_len, "page_size": w.page_size,
                   "mask": w.mask, "window": w.window, "rolling_buffer": w.rolling, "num_splits": splits,
                   "bytes_per_step": nbytes, "l2": "KV cache larger than L2 (no flush)"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": DECODE_NCU_TRAFFIC.get((w.name, decode_kernel_hash())),
                     "peak_source": f"{peak_src} hbm_gbs",
                     "note": "achieved over the whole step (decoding kernel plus split merge)"},
        "gpu_launches": args.steps * (2 if splits > 1 else 1),
        "launch_ms": {"median": statistics.median(per_step_ms), "best": min(per_step_ms)},
        "clocks": clk,
        "e2e": {"value": nbytes * e2e_steps / (e2e_ms / 1e3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
    }
    if not args.no_cpu_baseline:
        seqs = [0]
        dt, nb, threads = decode_cpu_sample(w, inp, seqs)
        line["cpu_baseline"] = {"value": nb / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
                                "sample": f"sequence 0 of the {w.name} workload, all heads "
                                          f"(fp64 NumPy, page-table gather and scores materialised), {dt:.1f} s"}
    print(json.dumps(line), flush=True)


RING_METRIC = "ring attention TFLOP/s (bf16, causal or window-adjusted; all ranks of the ring emulated on one GPU)"


def run_ring(args, w):
    """Ring attention with every rank emulated on one GPU, one after the other:
    each step runs all ranks' blocks through the forward kernel and their partial
    results through the merge kernel.  Shows what cutting the sequence into
    2R halves and merging costs against the single forward of the same workload
    (no communication happens on one GPU)."""
    from exact_io_aware_72_b200 import ring
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    R = args.ring_ranks
    q, k, v = make_qkv(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed, device=device, sharp=w.sharp)
    shares = ring.emulate_shares(q, k, v, R)
    del q, k, v
    flops = workload_flops(w, w.B)

    def eager_step():
        ring.run_emulated(shares, w.mask, w.scale, window=w.window)

    for _ in range(args.warmup):
        eager_step()
    torch.cuda.synchronize(device)
    stream = torch.cuda.current_stream(device)

    def timed(step):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
        evs[0].record(stream)
        for i in range(args.steps):
            step()
            evs[i + 1].record(stream)
        torch.cuda.synchronize(device)
        return [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)], evs[0].elapsed_time(evs[-1])

    eager_per, eager_ms = timed(eager_step)
    # The step's launches (one forward and one merge per block) captured once in a
    # CUDA graph and replayed: small blocks are otherwise bound by the host's
    # launch path, not by the GPU.
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            ring.run_emulated(shares, w.mask, w.scale, window=w.window)
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize(device)
        per, total_ms = timed(graph.replay)
    else:
        per, total_ms = eager_per, eager_ms
    peaks, peak_src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    blocks = sum(1 for r in range(R) for s in range(R) for a in ring.half_ids(R, r)
                 for b in ring.half_ids(R, (r - s) % R)
                 if ring.block_plan(a, b, w.mask, w.window, w.N // (2 * R)) is not None)
    achieved = flops / (statistics.mean(per) / 1e3) / 1e12
    line = {
        "metric": RING_METRIC, "pass": "ring", "value": flops * args.steps / (total_ms / 1e3) / 1e12,
        "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d, "mask": w.mask,
                   "ring_ranks": R, "block_rows": w.N // (2 * R), "blocks": blocks,
                   "launch": "cuda_graph" if graph is not None else "eager",
                   "l2": "inputs larger than L2 (no flush)"},
        "eager": {"value": flops * args.steps / (eager_ms / 1e3) / 1e12, "unit": "TFLOP/s",
                  "ms_per_step": eager_ms / args.steps},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "traffic": None, "peak_source": f"{peak_src} bf16_tflops (burst)"},
        "gpu_launches": 2 * blocks * args.steps,
        "launch_ms": {"median": statistics.median(per), "best": min(per)},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + sorted(DECODE_WORKLOADS), default=None,
                    help="default: long (fwd), dense (bwd, ring) or decode_gqa (decode)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--shape", default=None,
                    help="B,Hq,Hkv,N,d: run this shape instead of a named workload (profiling sweeps)")
    ap.add_argument("--mask", choices=["full", "causal", "sliding_window"], default=None)
    ap.add_argument("--window", type=int, default=None)
    ap.add_argument("--bwd-deterministic", action="store_true",
                    help="--pass bwd with d = 128: the two-kernel path (dq bitwise reproducible)")
    ap.add_argument("--pass", dest="which", choices=["fwd", "bwd", "decode", "ring"], default="fwd",
                    help="bwd: the backward pass; decode: a paged-KV decoding step; ring: ring attention with "
                         "its ranks emulated on one GPU (one GPU each)")
    ap.add_argument("--splits", type=int, default=0, help="decode: KV splits per sequence (0 = suggested)")
    ap.add_argument("--ring-ranks", type=int, default=8, help="ring: ranks emulated on the one GPU")
    ap.add_argument("--no-graph", action="store_true", help="ring: time eager launches only (no CUDA graph)")
    ap.add_argument("--dtype", choices=["bf16", "fp8"], default="bf16",
                    help="forward inputs: bf16, or E4M3 codes with per-tensor scales")
    ap.add_argument("--split", choices=["batch", "heads"], default="batch",
                    help="with N > 1 GPUs: every rank its own batch (weak scaling), or the workload's "
                         "(batch, KV-group) units split across ranks (strong scaling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.which == "decode":
        name = args.workload or "decode_gqa"
        if name not in DECODE_WORKLOADS:
            ap.error("--pass decode takes a decode_* workload")
        run_decode(args, DECODE_WORKLOADS[name])
        return
    if args.workload in DECODE_WORKLOADS:
        ap.error("decode_* workloads need --pass decode")
    w = WORKLOADS[args.workload or ("long" if args.which == "fwd" else "dense")]
    if args.shape or args.mask:
        from dataclasses import replace
        B, Hq, Hkv, N, d = (int(x) for x in args.shape.split(",")) if args.shape else (w.B, w.Hq, w.Hkv, w.N, w.d)
        mask = args.mask or w.mask
        w = replace(w, name="custom", B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, mask=mask,
                    window=args.window if mask == "sliding_window" else None, sharp=False)
    if args.impl == "reference":
        run_reference(args, w)
    elif args.which == "ring":
        run_ring(args, w)
    elif args.which == "bwd":
        run_backward(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
