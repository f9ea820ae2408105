#!/usr/bin/env python
"""Benchmark of the fused exact-attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step = one fused forward (one kernel launch) over the whole batch of the
workload, inputs resident in device memory.  The metric is attention-forward
TFLOP/s, counting 4*T^2*d_h per head and half of that when causal.  Prints ONE
JSON line (rank 0).

Default workload: B=4, H=32, T=8192, d_h=128, causal (the T >= 8192, d_h = 128
case the throughput target is quoted on).  Its Q/K/V (3 x 268 MB) are larger
than the 126 MB L2, so no L2 flush is needed between steps.

Multi-GPU (``torchrun --nproc-per-node N bench.py --gpus N``): heads are
independent, so every rank runs the whole workload on its own GPU with its own
seeded inputs and no data-path collective (weak scaling); the only collectives
are the timing barrier and the max over ranks of the step time.

``--impl reference`` times the float64 CPU oracle (the slow, obviously correct
program the kernel is checked against) on bounded row samples of the same
workload, on this host's cores, rank 0 only.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from attn_inputs import ORDER, WORKLOADS, make_qkv, bf16_bits  # noqa: E402

DEFAULT_WORKLOAD = "causal_T8192_d128"
METRIC = "attention fwd TFLOP/s on 1 B200 and % of dense BF16 tensor peak"
PEAK_FALLBACK = {"bf16_tflops": 1590.0, "hbm_gbs": 6650.0}
L2_BYTES = 126 << 20  # B200 L2
KERNEL_SOURCES = [os.path.join(ROOT, "exact_attention_124_b200", "csrc", f)
                  for f in ("fused_fwd.cuh", "sm100.cuh")]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip timing the other workloads (the per_config block)")
    ap.add_argument("--no-other-paths", action="store_true",
                    help="skip timing the backward, decode and unfused paths (the other_paths block)")
    ap.add_argument("--decode-tq", type=int, default=1, help="decode: new queries per head")
    ap.add_argument("--decode-hkv", type=int, default=0,
                    help="decode: K/V heads (0: the workload's H / 4)")
    ap.add_argument("--path", choices=["fused", "unfused", "backward", "decode"], default="fused",
                    help="unfused: the three-kernel materialised path (S and P in HBM); "
                         "backward: the gradient kernels (recomputing S and P); "
                         "decode: --decode-tq queries against a cache of the workload's T tokens")
    ap.add_argument("--batch", type=int, default=None, help="override the workload's B")
    ap.add_argument("--exp-split", type=int, default=None,
                    help="fused kernel variant: column pairs of every 8 whose exponentials run "
                         "on the FMA pipe (0, 2, 3, 4); default: the library's choice")
    args = ap.parse_args()
    if args.e2e_steps < 1 or args.steps < 1:
        ap.error("--steps and --e2e-steps must be at least 1")
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    return args


def workload_of(args):
    import dataclasses
    w = WORKLOADS[args.workload]
    if args.batch:
        w = dataclasses.replace(w, B=int(args.batch), name=f"{w.name}_B{int(args.batch)}")
    return w


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAK_FALLBACK), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the fused kernel from the committed ncu
    summary, or None when the summary is missing or the kernel changed since."""
    path = os.path.join(ROOT, "profiles", f"fused_fwd_{workload}.txt")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line:
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("kernel_source_sha256") != kernel_source_hash():
        return None
    try:
        return int(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.ok = [], 0, False
        self.period = period_s
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # pragma: no cover - NVML missing
            self.ok = False
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        nv = self.nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= int(get_r(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"],
                    "samples": 0}
        names = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def counted_flops(w) -> float:
    return w.flops()


def rank_seed(w, rank: int) -> int:
    """Each rank draws its own inputs: the workload's seed offset by 1000 * rank."""
    return w.seed + 1000 * rank


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Largest value of ``x`` over all ranks (the slowest rank sets the step
    time); a plain return when running alone."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank: float, world: int, ms_per_step: float) -> float:
    """Weak scaling: every rank does flops_per_rank per step; the job's step
    takes the slowest rank's time."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


# ---------------------------------------------------------------------------- CPU oracle
def oracle_sample(w, seconds: float, seed_offset: int = 0):
    """Time the float64 oracle on a sample of workload ``w`` sized to about
    ``seconds`` of CPU work: evenly spaced query rows of one head, and whole
    heads once one head is not enough.  Returns (TFLOP/s in the metric's
    counting, seconds, rows, threads, description)."""
    import numpy as np
    import oracle
    threads = oracle.default_threads()
    max_heads = min(w.heads, 64)
    q, k, v = make_qkv(1, max_heads, w.T, w.D, w.seed + seed_offset, w.qk_mult)
    qb, kb, vb = bf16_bits(q), bf16_bits(k), bf16_bits(v)

    def run(nheads, nrows):
        step = max(1, w.T // nrows)
        rows = np.arange(step // 2, w.T, step, dtype=np.int64)[:nrows]
        t0 = time.perf_counter()
        oracle.attn_fwd(qb, kb, vb, w.causal, w.scale, heads=np.arange(nheads), rows=rows,
                        nthreads=threads)
        dt = time.perf_counter() - t0
        # the metric's counting: 4*d per visible key (QK^T and PV), per row
        vis = (rows + 1) if w.causal else np.full(rows.shape, w.T)
        return rows, dt, float(4.0 * w.D * vis.sum()) * nheads

    nheads, n = 1, max(threads, 32)
    for _ in range(5):  # calibrate the sample size to the time budget
        rows, dt, fl = run(nheads, n)
        if dt >= 0.6 * seconds or (n >= w.T and nheads >= max_heads):
            break
        grow = seconds / max(dt, 1e-6)
        if n < w.T:
            n = int(min(w.T, max(n + 1, n * grow)))
        else:
            nheads = int(min(max_heads, max(nheads + 1, nheads * grow)))
    desc = (f"{len(rows)} evenly spaced query rows of {nheads} head(s) (T={w.T}, d_h={w.D}, "
            f"{'causal' if w.causal else 'full'}), float64, {threads} threads; FLOPs counted "
            f"as 4*d_h per visible key")
    return fl / dt / 1e12, dt, len(rows) * nheads, threads, desc


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    w = workload_of(args)
    per_step = max(1.0, min(args.cpu_seconds, 150.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup):
        oracle_sample(w, per_step / 4, seed_offset=i)
    vals, secs = [], []
    desc, threads = "", 0
    for i in range(args.steps):
        v, dt, nrows, threads, desc = oracle_sample(w, per_step, seed_offset=100 + i)
        vals.append(v)
        secs.append(dt)
    value = float(statistics.median(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * statistics.median(secs), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "shape": w.describe(), "seed": w.seed,
                   "note": "each step times a bounded row sample of the workload"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------- GPU arm
def run_ours(args):
    import torch
    import torch.distributed as dist
    import exact_attention_124_b200 as attn

    world, rank, local = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    w = workload_of(args)
    attn.load_library()
    if args.exp_split is not None:
        attn.set_exp_split(args.exp_split)
    peaks, peak_src = load_peaks()
    other = {"unfused": run_unfused, "backward": run_backward, "decode": run_decode}.get(args.path)
    if other is not None:
        rc = other(args, w, world, rank, local, peaks, peak_src)
        if world > 1:
            dist.destroy_process_group()
        return rc

    # inputs: per-rank seed, generated on the host, copied once (resident in HBM)
    q, k, v = make_qkv(w.B, w.H, w.T, w.D, rank_seed(w, rank), w.qk_mult)
    dev = torch.device("cuda", local)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o = torch.empty_like(qd)
    lse = torch.empty((w.B, w.H, w.T), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    per_launch, total_ms, clocks_main = time_fused(attn, w, qd, kd, vd, o, lse, stream, args.steps,
                                                   args.warmup, local, world)
    status = attn.last_error()
    launches = args.steps  # one fused kernel per step
    ms = max_over_ranks(total_ms / args.steps, world, dev)
    flops = counted_flops(w)
    value = whole_job_tflops(flops, world, ms)
    achieved = flops / (statistics.mean(per_launch) * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])

    # the other workloads, timed the same way on this GPU (rank 0 at N = 1 only)
    per_config = None
    if world == 1 and not args.no_per_config and args.workload == DEFAULT_WORKLOAD:
        per_config = {}
        for name in ORDER:
            if name == w.name:
                continue
            per_config[name] = time_other(attn, WORKLOADS[name], dev, stream, args, local, peaks)
            status |= attn.last_error()

    # the other paths of the library on the same GPU, each timed like its own
    # --path mode (backward and decode on this workload's shape; the unfused
    # path on the two workloads whose S and P fit in a few GB)
    other_paths = None
    if world == 1 and not args.no_other_paths and args.workload == DEFAULT_WORKLOAD:
        import argparse as _ap
        sub = _ap.Namespace(**vars(args))
        sub.steps, sub.warmup = max(3, min(args.steps, 10)), 3
        other_paths = {"backward": run_backward(sub, w, 1, rank, local, peaks, peak_src, emit=False),
                       "decode": run_decode(sub, w, 1, rank, local, peaks, peak_src, emit=False)}
        for name in ("causal_T4096_d64", "full_T2048_d128_qk4"):
            other_paths["unfused_" + name] = run_unfused(sub, WORKLOADS[name], 1, rank, local, peaks,
                                                         peak_src, emit=False)
        status |= attn.last_error()

    # end to end through the host-buffer C-ABI entry point
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty((w.B, w.H, w.T), dtype=torch.float32).pin_memory()
    for _ in range(1):
        attn.fwd_host(qh, kh, vh, oh, lh, qd, kd, vd, o, lse, w.causal, w.scale, stream=stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.e2e_steps):
        attn.fwd_host(qh, kh, vh, oh, lh, qd, kd, vd, o, lse, w.causal, w.scale, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, world, dev)
    status |= attn.last_error()
    h2d = 3 * q.numel() * 2
    d2h = o.numel() * 2 + lse.numel() * 4

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v_cpu, dt, nrows, threads, desc = oracle_sample(w, args.cpu_seconds)
        cpu = {"value": v_cpu, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": desc, "seconds": round(dt, 2)}

    if rank == 0:
        clocks = clocks_main
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "shape": w.describe(), "global_batch": w.B * world,
                       "heads": w.H, "seq_len": w.T, "d_h": w.D, "causal": w.causal,
                       "seed": w.seed, "parallelism": f"heads{world}" if world > 1 else "single",
                       "l2": "inputs larger than L2 (Q/K/V 3 x %.0f MB); no flush" %
                             (q.numel() * 2 / 1e6),
                       "flops_per_step_per_gpu": flops,
                       "grid_ctas": attn.fused_grid_ctas(w.B, w.H, w.T, w.D, w.causal)},
            "pct_of_peak": 100.0 * value / world / peak,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak,
                         "peak_source": f"{peak_src} bf16_tflops (cuBLAS bf16 burst)",
                         "frac_of_sustained": achieved / float(peaks.get(
                             "bf16_tflops_sustained", peak)),
                         "frac_of_datasheet_2250": achieved / 2250.0,
                         "traffic": profiled_traffic(w.name),
                         "algorithmic_bytes": (3 * q.numel() + o.numel()) * 2 + lse.numel() * 4,
                         "launch_ms_mean": statistics.mean(per_launch),
                         "launch_ms_min": min(per_launch)},
            "clocks": clocks,
            "per_config": per_config,
            "other_paths": other_paths,
            "gpu_launches": launches,
            "e2e": {"value": whole_job_tflops(flops, world, e2e_ms), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms, "api": "attn_fwd_host"},
            "cpu_baseline": cpu,
            "device_status": status,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0 if status == 0 else 1


def time_fused(attn, w, qd, kd, vd, o, lse, stream, steps, warmup, local, world, flush=None):
    """W untimed launches, then K launches with CUDA events around each on the
    launching stream and NVML clock sampling meanwhile.  With ``flush`` (a
    device buffer larger than L2) the buffer is rewritten before every launch,
    outside the events.  Returns (per-launch ms, first-to-last ms, clocks)."""
    import torch
    import torch.distributed as dist

    def step():
        attn.fwd(qd, kd, vd, w.causal, w.scale, o=o, lse=lse, stream=stream)

    for _ in range(max(3, warmup)):
        step()
    if attn.last_error() != 0:
        raise SystemExit(f"device error during warm-up ({w.name})")
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * steps)]
    sampler = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    for i in range(steps):
        if flush is not None:
            flush.zero_()
        ev[2 * i].record(stream)
        step()
        ev[2 * i + 1].record(stream)
    torch.cuda.synchronize()
    sampler.stop()
    if world > 1:
        dist.barrier()
    per_launch = [ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(steps)]
    total = ev[0].elapsed_time(ev[-1]) if flush is None else sum(per_launch)
    return per_launch, total, sampler.summary()


def time_other(attn, w, dev, stream, args, local, peaks):
    """One entry of the bench line's per_config block: workload ``w`` timed
    like the headline (inputs resident; L2 rewritten before each launch when
    the inputs would fit in it)."""
    import torch
    q, k, v = make_qkv(w.B, w.H, w.T, w.D, w.seed, w.qk_mult)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    del q, k, v
    o = torch.empty_like(qd)
    lse = torch.empty((w.B, w.H, w.T), dtype=torch.float32, device=dev)
    in_bytes = 3 * qd.numel() * 2
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if in_bytes < (256 << 20) else None
    per_launch, _, clocks = time_fused(attn, w, qd, kd, vd, o, lse, stream, args.steps,
                                       args.warmup, local, 1, flush)
    mean_ms = statistics.mean(per_launch)
    tf = counted_flops(w) / (mean_ms * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    out = {"shape": w.describe(), "seed": w.seed, "ms_mean": mean_ms, "ms_min": min(per_launch),
           "tflops": tf, "frac": tf / peak, "frac_of_datasheet_2250": tf / 2250.0,
           "l2": ("256 MB rewritten before each launch" if flush is not None else
                  "inputs larger than L2 (%.0f MB); no flush" % (in_bytes / 1e6)),
           "grid_ctas": attn.fused_grid_ctas(w.B, w.H, w.T, w.D, w.causal), "launches": args.steps,
           "clocks": clocks}
    del qd, kd, vd, o, lse, flush
    torch.cuda.empty_cache()
    return out


def unfused_bytes(w) -> int:
    """Algorithmic HBM bytes of the materialised path per step: S written and
    read, P written and read (bf16; T^2 entries per head, or under the causal
    mask the 128 x 128 tiles at or below the diagonal, which is all the path
    moves), plus Q, K, V read (K1 reads Q and K, K3 reads V), O written (bf16)
    and lse written (fp32)."""
    heads = w.B * w.H
    nt = w.T // 128
    entries = (nt * (nt + 1) // 2) * 128 * 128 if w.causal else w.T * w.T
    return heads * (4 * entries * 2 + 4 * w.T * w.D * 2 + w.T * 4)


def run_unfused(args, w, world, rank, local, peaks, peak_src, emit=True):
    import torch
    import exact_attention_124_b200 as attn
    dev = torch.device("cuda", local)
    q, k, v = [t.to(dev) for t in make_qkv(w.B, w.H, w.T, w.D, rank_seed(w, rank), w.qk_mult)]
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.T), dtype=torch.float32, device=dev)
    S = torch.empty((w.B, w.H, w.T, w.T), dtype=torch.bfloat16, device=dev)
    P = torch.empty_like(S)
    stream = torch.cuda.current_stream()

    def step():
        attn.fwd_unfused(q, k, v, w.causal, w.scale, o=o, lse=lse, s_ws=S, p_ws=P, stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    if attn.last_error() != 0:
        raise SystemExit("device error during warm-up")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    torch.cuda.synchronize()
    sampler.start()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    sampler.stop()
    status = attn.last_error()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    nbytes = unfused_bytes(w)
    gbs = nbytes / (ms * 1e-3) / 1e9
    hbm = float(peaks["hbm_gbs"])
    if not emit:
        del S, P
        torch.cuda.empty_cache()
        return {"workload": w.name, "shape": w.describe(), "ms_per_step": ms,
                "tflops": counted_flops(w) / (ms * 1e-3) / 1e12, "gbs": gbs, "frac_of_hbm": gbs / hbm,
                "algorithmic_bytes": nbytes, "launches": 3 * args.steps,
                "clocks": sampler.summary(), "device_status": status}
    if rank == 0:
        line = {
            "metric": METRIC + " (unfused three-kernel path)", "path": "unfused",
            "value": whole_job_tflops(counted_flops(w), world, ms), "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "shape": w.describe(), "seed": w.seed,
                       "workspace_bytes": 2 * S.numel() * 2},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                         "frac": gbs / hbm, "peak_source": f"{peak_src} hbm_gbs",
                         "algorithmic_bytes": nbytes, "traffic": None},
            "clocks": sampler.summary(), "gpu_launches": 3 * args.steps,
            "device_status": status,
        }
        print(json.dumps(line), flush=True)
    return 0 if status == 0 else 1


def run_backward(args, w, world, rank, local, peaks, peak_src, emit=True):
    """Times attn_bwd (row statistics + dK/dV kernel + dQ kernel) per step.
    Counted FLOPs: 10*T^2*d_h per head (five T x T x d_h products: S, dP, dV,
    dK, dQ), halved when causal; the kernels actually run seven (S and dP are
    recomputed once per gradient kernel), reported beside it."""
    import torch
    import exact_attention_124_b200 as attn
    dev = torch.device("cuda", local)
    q, k, v = [t.to(dev) for t in make_qkv(w.B, w.H, w.T, w.D, rank_seed(w, rank), w.qk_mult)]
    g = make_qkv(w.B, w.H, w.T, w.D, rank_seed(w, rank) + 7)[0].to(dev)
    o, lse = attn.fwd(q, k, v, w.causal, w.scale)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(int(attn.load_library().attn_bwd_workspace_bytes(w.B, w.H, w.T)),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        attn.bwd(q, k, v, o, lse, g, w.causal, w.scale, dq=dq, dk=dk, dv=dv, ws=ws, stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    if attn.last_error() != 0:
        raise SystemExit("device error during warm-up")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    torch.cuda.synchronize()
    sampler.start()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    sampler.stop()
    status = attn.last_error()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    counted = 2.5 * counted_flops(w)
    peak = float(peaks["bf16_tflops"])
    if not emit:
        tf = counted / (ms * 1e-3) / 1e12
        return {"workload": w.name, "shape": w.describe(), "ms_per_step": ms, "tflops_counted": tf,
                "frac": tf / peak, "tflops_executed": 1.4 * tf, "launches": 3 * args.steps,
                "clocks": sampler.summary(), "device_status": status}
    if rank == 0:
        value = whole_job_tflops(counted, world, ms)
        line = {
            "metric": "attention bwd TFLOP/s (10*T^2*d_h per head, halved causal)",
            "path": "backward", "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "shape": w.describe(), "seed": w.seed},
            "roofline": {"bound": "tensor", "achieved": value / world, "peak": peak,
                         "unit": "TFLOP/s", "frac": value / world / peak,
                         "peak_source": f"{peak_src} bf16_tflops",
                         "executed_tflops": 1.4 * value / world},
            "clocks": sampler.summary(), "gpu_launches": 3 * args.steps, "device_status": status,
        }
        print(json.dumps(line), flush=True)
    return 0 if status == 0 else 1


def run_decode(args, w, world, rank, local, peaks, peak_src, emit=True):
    """Times attn_fwd_decode (split-KV partials + merge): --decode-tq queries
    per head against a K/V cache of the workload's T tokens with H_kv heads.
    HBM-bound: algorithmic bytes = the K/V cache read once + Q read + O, lse
    written."""
    import torch
    import exact_attention_124_b200 as attn
    dev = torch.device("cuda", local)
    H_kv = args.decode_hkv or max(1, w.H // 4)
    Tq, Tk = args.decode_tq, w.T
    q = make_qkv(w.B, w.H, Tq, w.D, rank_seed(w, rank))[0].to(dev)
    _, k, v = make_qkv(w.B, H_kv, Tk, w.D, rank_seed(w, rank) + 1)
    k, v = k.to(dev), v.to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, Tq), dtype=torch.float32, device=dev)
    lib = attn.load_library()
    ws = torch.empty(int(lib.attn_decode_workspace_bytes(w.B, w.H, H_kv, Tq, Tk, w.D, 0)),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        attn.fwd_decode(q, k, v, True, w.scale, splits=0, o=o, lse=lse, ws=ws, stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    if attn.last_error() != 0:
        raise SystemExit("device error during warm-up")
    # Between steps: write a buffer larger than L2 (evicts the cache from L2), then
    # read a second one, so that the lines left in L2 are clean and the timed
    # kernel pays no write-back of the flush's dirty lines.
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_rd = torch.zeros(256 << 20, dtype=torch.uint8, device=dev)
    flush_sink = torch.empty((), dtype=torch.int64, device=dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    sampler = ClockSampler(local)
    torch.cuda.synchronize()
    sampler.start()
    for a, b in evs:
        flush.zero_()
        torch.sum(flush_rd, dim=0, dtype=torch.int64, out=flush_sink)
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize()
    sampler.stop()
    status = attn.last_error()
    # the mean, not the median: at tens of microseconds the event timestamps
    # come in steps of about 2 us, and only the mean of many steps resolves
    # differences below one step
    ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in evs), world, dev)
    nbytes = 2 * k.numel() * 2 + q.numel() * 2 + o.numel() * 2 + lse.numel() * 4
    gbs = nbytes / (ms * 1e-3) / 1e9
    hbm = float(peaks["hbm_gbs"])
    # Second figure: steps back to back with no flush, one pair of events around
    # all of them, so each launch's set-up overlaps the step before it (as in a
    # decode loop; the single-step figure above includes the whole launch
    # latency after the flush kernels).  Only when the cache is larger than L2,
    # so that every step reads it from DRAM again.
    cache_bytes = 2 * k.numel() * 2
    pipelined = None
    if cache_bytes > L2_BYTES:
        nb = max(10, args.steps)
        for _ in range(3):
            step()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(nb):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        status = status or attn.last_error()
        pms = max_over_ranks(e0.elapsed_time(e1) / nb, world, dev)
        pg = nbytes / (pms * 1e-3) / 1e9
        pipelined = {"us_per_step": 1e3 * pms, "gbs": pg, "frac_of_hbm": pg / hbm, "steps": nb,
                     "l2": f"no flush: the {cache_bytes / 2**20:.0f} MiB cache is larger than the "
                           f"{L2_BYTES / 2**20:.0f} MiB L2"}
    # Third figure: the isolated step of the first figure (same flush before each
    # step, same events) replayed from a CUDA graph that holds its two launches,
    # as a decode loop would run it; the host-side launch path is then off the
    # timed critical path.
    # (A failed capture is reported in this entry and does not end the run.)
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    try:
        with torch.cuda.graph(g):
            attn.fwd_decode(q, k, v, True, w.scale, splits=0, o=o, lse=lse, ws=ws)
        captured = None
    except Exception as e:  # noqa: BLE001 -- reported, not hidden
        captured = f"{type(e).__name__}: {e}".splitlines()[0][:200]
    torch.cuda.synchronize()
    if captured is None:
        for _ in range(3):
            g.replay()
        gevs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(args.steps)]
        torch.cuda.synchronize()
        for a, b in gevs:
            flush.zero_()
            torch.sum(flush_rd, dim=0, dtype=torch.int64, out=flush_sink)
            a.record(stream)
            g.replay()
            b.record(stream)
        torch.cuda.synchronize()
        status = status or attn.last_error()
        gms = statistics.mean(a.elapsed_time(b) for a, b in gevs)
    else:
        gms = float("nan")
    # every rank takes the same collective step, captured or not
    gms = max_over_ranks(gms, world, dev)
    gg = nbytes / (gms * 1e-3) / 1e9
    graphed = {"us_per_step": 1e3 * gms, "gbs": gg, "frac_of_hbm": gg / hbm, "steps": args.steps,
               "l2": "256 MB written, then 256 MB read, before each step"}
    if captured is not None:
        graphed = {"error": captured}
    del g
    if not emit:
        return {"workload": f"decode B={w.B} H={w.H} H_kv={H_kv} Tq={Tq} Tk={Tk} d_h={w.D} causal",
                "us_per_step": 1e3 * ms, "gbs": gbs, "frac_of_hbm": gbs / hbm,
                "algorithmic_bytes": nbytes, "launches": 2 * args.steps,
                "l2": "256 MB written, then 256 MB read, before each step",
                "pipelined": pipelined, "graph": graphed,
                "clocks": sampler.summary(), "device_status": status}
    if rank == 0:
        line = {
            "metric": "attention decode: effective HBM GB/s (K/V cache read once)",
            "path": "decode", "value": gbs * world, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": f"decode B={w.B} H={w.H} H_kv={H_kv} Tq={Tq} Tk={Tk} "
                                   f"d_h={w.D} causal", "l2": "256 MB written, then 256 MB read, before each step"},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                         "frac": gbs / hbm, "peak_source": f"{peak_src} hbm_gbs",
                         "algorithmic_bytes": nbytes},
            "pipelined": pipelined, "graph": graphed,
            "clocks": sampler.summary(), "gpu_launches": 2 * args.steps, "device_status": status,
        }
        print(json.dumps(line), flush=True)
    return 0 if status == 0 else 1


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
