"""Benchmark of the fused exact-attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one fa_fwd launch over the whole problem (every query row of
every head).  The default problem is B=2, H=16, N=8192, d=128, causal, bf16
inputs from N(0,1) with seed 2; inputs plus output (268 MB) exceed the 126 MB
L2, so no flush is inserted between steps.  FLOPs are counted as
4*B*H*N^2*d, halved for causal.

Timing: W untimed warm-up steps, then exactly K steps bracketed by a barrier
and a device synchronise on both sides, measured with CUDA events on the
launching stream; the time is the maximum over ranks.  With N > 1 (launched
by torch.distributed.run) every rank runs the same problem on its own seeded
inputs: weak scaling with no collective on the data path.

Rank 0 prints one JSON line.  ``--impl reference`` times the float64 CPU
oracle instead (the reference arm), on bounded row samples of the same
problem; under torchrun only rank 0 runs it.
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

METRIC = "attention fwd TFLOP/s (bf16, 1×B200) and % of dense-BF16 tensor peak"
DEFAULT_WORKLOAD = "b2h16n8192d128_causal"
FALLBACK_PEAK_TFLOPS = 1590.0
FALLBACK_PEAK_SUSTAINED_TFLOPS = 1400.0
L2_BYTES = 126 * 1024 * 1024
KERNEL_SOURCES = ["exact_softmax_attention_02_b200/csrc/fa_fwd.cu",
                  "exact_softmax_attention_02_b200/csrc/sm100.cuh"]


# ---------------------------------------------------------------------------
# distributed plumbing (host logic, covered by CPU gloo tests)
# ---------------------------------------------------------------------------

def dist_env():
    """(rank, local_rank, world_size) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def init_dist(world: int, backend: str):
    import datetime

    import torch.distributed as dist

    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def rank_seed(seed: int, rank: int) -> int:
    """Each rank draws its own inputs; rank 0 keeps the workload's seed."""
    return seed + 7919 * rank


def max_over_ranks(value: float, dist, device=None) -> float:
    import torch

    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, dist, device=None) -> float:
    import torch

    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def weak_scaling_value(flops_per_rank_step: float, world: int, steps: int, seconds: float) -> float:
    """Whole-job TFLOP/s: all ranks' FLOPs over the slowest rank's time."""
    return flops_per_rank_step * world * steps / seconds / 1e12


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only; no setting is changed)
# ---------------------------------------------------------------------------

_REASON_BITS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
    0x100: "display_clock_setting",
}


class ClockSampler:
    """Polls SM clock, power and clock-event reasons from a thread."""

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._nvml = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # NVML unavailable: report no clocks rather than guess
            self._nvml = None

    def _run(self):
        n = self._nvml
        while not self._stop.is_set():
            try:
                mhz = n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM)
                try:
                    reasons = n.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except Exception:
                    reasons = n.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                util = n.nvmlDeviceGetUtilizationRates(self._h).gpu
                self.samples.append((mhz, int(reasons), util))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self._nvml is not None and self.period > 0:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        loaded = [s for s in self.samples if not (s[1] & 0x1)] or self.samples
        mask = 0
        for _, r, _ in loaded:
            mask |= r
        reasons = [name for bit, name in sorted(_REASON_BITS.items()) if mask & bit and bit != 0x1]
        return {"sm_mhz": statistics.median(s[0] for s in loaded), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(loaded)}


# ---------------------------------------------------------------------------
# peaks and committed ncu evidence
# ---------------------------------------------------------------------------

def tensor_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            peaks = json.load(f)
        return float(peaks["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops, burst)"
    except Exception:
        return FALLBACK_PEAK_TFLOPS, "fallback (1.59 PFLOP/s, earlier measurement on this pool)"


def tensor_peak_sustained():
    """The bf16 peak for a kernel timed inside a seconds-long loop under the
    power cap (MEASURED_PEAKS.json bf16_tflops_sustained), else the pool's
    earlier figure (about 1.4 PFLOP/s at about 1.3 GHz)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            peaks = json.load(f)
        return float(peaks["bf16_tflops_sustained"]), "measured (MEASURED_PEAKS.json bf16_tflops_sustained)"
    except Exception:
        return FALLBACK_PEAK_SUSTAINED_TFLOPS, "fallback (1.4 PFLOP/s sustained, earlier measurement on this pool)"


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except Exception:
        return 6650.0, "fallback (6.65 TB/s, earlier measurement on this pool)"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def committed_traffic(workload: str):
    """DRAM bytes per launch from the committed ncu summary for this workload,
    or None when there is none or the kernel source changed since."""
    path = os.path.join(ROOT, "profiles", f"fa_fwd_{workload}_ncu.md")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            line = line.strip().lstrip("-* ")
            for key in ("dram_bytes_per_launch", "kernel_source_sha256"):
                if line.startswith(key + ":"):
                    rest = line.split(":", 1)[1].split()
                    vals[key] = rest[0].strip("`") if rest else ""
    if vals.get("kernel_source_sha256") != kernel_source_hash():
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------------------
# the oracle on host cores (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------

def blas_threads() -> int:
    try:
        import threadpoolctl

        info = threadpoolctl.threadpool_info()
        n = [i["num_threads"] for i in info if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample_time(w, q32, k32, v32, rows):
    """Run the oracle on ``rows``; return (seconds, counted FLOPs)."""
    from oracle import attention_rows, flops_for_rows

    t0 = time.perf_counter()
    attention_rows(q32, k32, v32, w.scale, w.causal, rows)
    dt = time.perf_counter() - t0
    return dt, flops_for_rows(rows, w.N, w.d, w.causal)


def oracle_inputs(w, seed):
    from exact_softmax_attention_02_b200.inputs import make_qkv

    q, k, v = make_qkv(w.B, w.H, w.N, w.d, seed, w.q_std)
    return q.float().numpy(), k.float().numpy(), v.float().numpy()


def random_rows(w, count, seed):
    import numpy as np

    rng = np.random.default_rng(seed)
    flat = rng.choice(w.B * w.H * w.N, size=min(count, w.B * w.H * w.N), replace=False)
    return np.stack([flat // (w.H * w.N), (flat // w.N) % w.H, flat % w.N], axis=1)


def cpu_baseline(w, seed, target_s: float = 12.0):
    """Oracle throughput on a bounded random row sample, in TFLOP/s."""
    q32, k32, v32 = oracle_inputs(w, seed)
    total = w.B * w.H * w.N
    n = 64
    # grow the sample until one timed pass takes at least half the target
    for attempt in range(8):
        rows = random_rows(w, n, seed + 2 + attempt)
        dt, flops = oracle_sample_time(w, q32, k32, v32, rows)
        if dt >= 0.5 * target_s or n >= total:
            break
        n = int(min(total, n * min(16.0, max(2.0, target_s / max(dt, 1e-3)))))
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"{len(rows)} random query rows of {w.name} (float64 numpy, "
                      f"{dt:.1f} s; FLOPs counted 4*d per allowed key)"}


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------

def run_reference(args, w):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    q32, k32, v32 = oracle_inputs(w, w.seed)
    budget_per_step = min(args.ref_step_seconds, 150.0 / max(1, args.steps + args.warmup))
    n = 32
    dt, _ = oracle_sample_time(w, q32, k32, v32, random_rows(w, n, 1))
    n = int(max(8, min(w.B * w.H * w.N, n * budget_per_step / max(dt, 1e-3))))
    for i in range(args.warmup):
        oracle_sample_time(w, q32, k32, v32, random_rows(w, n, 100 + i))
    tot_t, tot_f = 0.0, 0.0
    for i in range(args.steps):
        dt, fl = oracle_sample_time(w, q32, k32, v32, random_rows(w, n, 1000 + i))
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    sample = (f"{n} random query rows of {w.name} per step (float64 numpy oracle; "
              f"FLOPs counted 4*d per allowed key)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {**w.as_config(), "l2": "host oracle (no GPU)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# The other configurations the target names, measured in the same run as the
# headline (one GPU only): the d=64 problem, the two long-context causal
# problems, and the backward pass of the headline problem.
EXTRA_CONFIGS = [
    ("b4h16n4096d64", "forward"),
    ("b1h32n32768d128_causal_q4", "forward"),
    ("b1h8n131072d128_causal", "forward"),
    ("b2h16n8192d128_causal", "backward"),
]


def measure_config(name: str, path: str, dev, steps: int = 20, warmup: int = 5):
    """Kernel throughput of one more configuration: W untimed launches, then
    K launches timed with CUDA events on the launching stream, clocks sampled
    during the timed launches.  Returns a dict for the bench line."""
    import torch

    from exact_softmax_attention_02_b200 import fa
    from exact_softmax_attention_02_b200.inputs import WORKLOADS, make_workload_inputs

    w = WORKLOADS[name]
    q, k, v = (t.to(dev) for t in make_workload_inputs(w))
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    flops = w.flops
    if path == "backward":
        fa.fa_fwd(q, k, v, o, lse, scale=w.scale, causal=w.causal, stream=stream)
        g = torch.Generator(device="cpu").manual_seed(w.seed + 100)
        do = torch.randn(q.shape, generator=g).to(torch.bfloat16).to(dev)
        grads = [torch.empty_like(q) for _ in range(3)]
        ws = torch.empty(max(16, fa.bwd_workspace_bytes(w.B, w.H, w.N)), dtype=torch.uint8, device=dev)
        flops *= 2.5  # five N^2 d products against the forward's two

        def step():
            fa.fa_bwd(q, k, v, o, do, lse, *grads, workspace=ws, scale=w.scale, causal=w.causal,
                      stream=stream)
    else:
        def step():
            fa.fa_fwd(q, k, v, o, lse, scale=w.scale, causal=w.causal, stream=stream)

    for _ in range(warmup):
        step()
    if fa.device_status(stream) != 0:
        raise RuntimeError(f"{name} {path}: kernel reported a device failure in warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    sampler = ClockSampler(dev.index, period_s=float(os.environ.get("FA_BENCH_CLOCK_PERIOD", "0.01")))
    sampler.start()
    torch.cuda.synchronize(dev)
    for a, b in ev:
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize(dev)
    sampler.stop()
    if fa.device_status(stream) != 0:
        raise RuntimeError(f"{name} {path}: kernel reported a device failure")
    ms = sorted(a.elapsed_time(b) for a, b in ev)
    mean_s = sum(ms) / len(ms) / 1e3
    peak, _ = tensor_peak()
    peak_s, _ = tensor_peak_sustained()
    tf = flops / mean_s / 1e12
    # frac: against the burst peak; frac_sustained: against the peak a
    # seconds-long loop holds under the power cap, the fair one for the long
    # configurations (their timed loop lasts about a second)
    out = {"path": path, "tflops": tf, "frac": tf / peak, "frac_sustained": tf / peak_s,
           "ms_per_step": 1e3 * mean_s,
           "ms_min": ms[0], "ms_median": ms[len(ms) // 2], "steps": steps, "warmup": warmup,
           "flops_per_step": flops, "clocks": sampler.summary(),
           "kernel": ("bwd_rowdot + bwd_dkdv_kernel + bwd_dq_convert" if path == "backward"
                      else f"fa_fwd_kernel<{w.d},{str(w.causal).lower()}>"),
           "launches": steps * (3 if path == "backward" else 1)}
    if path == "backward":
        out["flops_convention"] = "2.5 x forward (five N^2 d products)"
    del q, k, v, o, lse
    torch.cuda.empty_cache()
    return out


def run_ours(args, w):
    import torch

    from exact_softmax_attention_02_b200 import fa
    from exact_softmax_attention_02_b200.inputs import make_qkv

    rank, local_rank, world = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (B200); the CPU oracle arm is --impl reference")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = init_dist(world, "nccl")

    seed = rank_seed(w.seed, rank)
    q_h, k_h, v_h = make_qkv(w.B, w.H, w.N, w.d, seed, w.q_std)
    q, k, v = (t.to(dev) for t in (q_h, k_h, v_h))
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    splits = None
    launches_per_step = 1
    std_events = None
    if args.path == "standard":
        from exact_softmax_attention_02_b200 import comparator

        g = min(w.B * w.H, comparator.heads_per_group(w.N))
        std_buffers = (torch.empty((g, w.N, w.N), dtype=torch.float32, device=dev),
                       torch.empty((g, w.N, w.N), dtype=torch.bfloat16, device=dev))
        launches_per_step = (w.B * w.H + g - 1) // g  # our softmax; the two GEMMs are cuBLAS'
    bwd = None
    if args.path == "backward":
        # one forward for O and LSE, then every step is one fa_bwd
        fa.fa_fwd(q, k, v, o, lse, scale=w.scale, causal=w.causal, stream=stream)
        g = torch.Generator(device="cpu").manual_seed(w.seed + 100)
        do = torch.randn(q.shape, generator=g).to(torch.bfloat16).to(dev)
        bwd = dict(do=do, dq=torch.empty_like(q), dk=torch.empty_like(q), dv=torch.empty_like(q),
                   ws=torch.empty(max(16, fa.bwd_workspace_bytes(w.B, w.H, w.N)), dtype=torch.uint8,
                                  device=dev))
        launches_per_step = 3  # D = rowsum(dO*O), dK/dV, dQ
    if args.path == "splitkv":
        splits = args.splits if args.splits > 0 else fa.splitkv_default_splits(w.B, w.H, w.N, w.d, w.causal)
        ws = torch.empty(max(16, fa.splitkv_workspace_bytes(w.B, w.H, w.N, w.d, splits, w.causal)),
                         dtype=torch.uint8, device=dev)
        launches_per_step = 1 if splits == 1 else 2  # split kernel + merge

    def step():
        if bwd is not None:
            fa.fa_bwd(q, k, v, o, bwd["do"], lse, bwd["dq"], bwd["dk"], bwd["dv"], workspace=bwd["ws"],
                      scale=w.scale, causal=w.causal, stream=stream)
        elif args.path == "standard":
            comparator.standard_attention(q, k, v, o, lse, scale=w.scale, causal=w.causal,
                                          buffers=std_buffers, softmax_events=std_events)
        elif splits is None:
            fa.fa_fwd(q, k, v, o, lse, scale=w.scale, causal=w.causal, stream=stream)
        else:
            fa.fa_fwd_splitkv(q, k, v, o, lse, workspace=ws, num_splits=splits, scale=w.scale,
                              causal=w.causal, stream=stream)

    for _ in range(args.warmup):
        step()
    if fa.device_status(stream) != 0:
        raise RuntimeError("kernel reported a device timeout during warm-up")

    sampler = ClockSampler(local_rank, period_s=float(os.environ.get("FA_BENCH_CLOCK_PERIOD", "0.01")))
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler.start()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    if args.path == "standard":
        std_events = []
    # the timed region: K steps between two events on the launching stream
    # (no event between steps, so small problems are not charged for them)
    t_start.record(stream)
    for _ in range(args.steps):
        step()
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    sampler.stop()
    if fa.device_status(stream) != 0:
        raise RuntimeError("kernel reported a device timeout in the timed region")
    elapsed = t_start.elapsed_time(t_end) / 1e3
    elapsed_max = max_over_ranks(elapsed, dist, dev)
    # device time per step over the timed region: the launches are queued
    # back to back, so this is the average launch duration (all kernels of a
    # step together when a step has several)
    avg_launch_s = elapsed_max / args.steps
    # the spread of single launches, from a separate untimed pass with an
    # event pair around each step (the comparator's softmax events stay those
    # of the timed region)
    std_timed, std_events = std_events, None
    n_spread = min(args.steps, 30)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_spread)]
    for a, b in ev:
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize(dev)
    launch_ms = [a.elapsed_time(b) for a, b in ev]

    # end to end through the public API: pinned host inputs -> device -> O, LSE back to host
    o_h = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    lse_h = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    q_p, k_p, v_p = (t.pin_memory() for t in (q_h, k_h, v_h))
    if bwd is not None:
        o_hb = o.cpu().pin_memory()
        do_hb = bwd["do"].cpu().pin_memory()
        lse_hb = lse.cpu().pin_memory()
        grads_h = [torch.empty(q.shape, dtype=q.dtype, pin_memory=True) for _ in range(3)]
    e2e_steps = max(3, min(args.steps, 20))
    def api_call():
        if bwd is not None:
            # end to end: host q, k, v, o, do, lse in; dq, dk, dv back to the host
            dev_t = [t.to(dev, non_blocking=True) for t in (q_p, k_p, v_p, o_hb, do_hb)]
            l_d = lse_hb.to(dev, non_blocking=True)
            g_d = [torch.empty_like(dev_t[0]) for _ in range(3)]
            fa.fa_bwd(*dev_t[:4], dev_t[4], l_d, *g_d, scale=w.scale, causal=w.causal)
            for hbuf, dbuf in zip(grads_h, g_d):
                hbuf.copy_(dbuf, non_blocking=True)
            torch.cuda.current_stream(dev).synchronize()
        elif args.path == "standard":
            qd, kd, vd = (t.to(dev, non_blocking=True) for t in (q_p, k_p, v_p))
            od, ld = comparator.standard_attention(qd, kd, vd, scale=w.scale, causal=w.causal,
                                                   buffers=std_buffers)
            o_h.copy_(od, non_blocking=True)
            lse_h.copy_(ld, non_blocking=True)
            torch.cuda.current_stream(dev).synchronize()
        else:
            fa.attention_forward(q_p, k_p, v_p, scale=w.scale, causal=w.causal, out=(o_h, lse_h),
                                 num_splits=splits)

    for _ in range(2):
        api_call()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        api_call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_s = max_over_ranks(e0.elapsed_time(e1) / 1e3, dist, dev)
    h2d = 3 * q.numel() * q.element_size()
    d2h = o.numel() * o.element_size() + lse.numel() * lse.element_size()
    if bwd is not None:
        h2d = 5 * q.numel() * q.element_size() + lse.numel() * lse.element_size()
        d2h = 3 * q.numel() * q.element_size()

    clocks = sampler.summary()
    # backward: five N^2 d products (2.5x the forward's two), the usual count
    flops = w.flops * (2.5 if bwd is not None else 1.0)
    value = weak_scaling_value(flops, world, args.steps, elapsed_max)
    peak, peak_src = tensor_peak()
    achieved = flops / avg_launch_s / 1e12
    traffic = committed_traffic(w.name)
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic, "peak_source": peak_src,
                "kernel": f"fa_fwd_kernel<{w.d},{str(w.causal).lower()}>"
                          + (" + fa_merge_kernel" if args.path == "splitkv" and launches_per_step == 2 else ""),
                "kernel_source_sha256": kernel_source_hash()}
    if bwd is not None:
        # one step = rowdot + dK/dV + dQ kernels, timed together
        roofline.update(kernel="bwd_rowdot + bwd_dkdv_kernel + bwd_dq_convert", traffic=None,
                        flops_convention="2.5 x forward (five N^2 d products)")
    if args.path == "standard":
        # the comparator's dominant kernel is the HBM-bound row softmax:
        # it reads the fp32 scores and writes the bf16 probabilities and LSE
        sm_ms = [a.elapsed_time(b) for a, b in std_timed]
        sm_s = max_over_ranks(sum(sm_ms) / 1e3 / args.steps, dist, dev)
        nbytes = w.B * w.H * w.N * (6 * w.N + 4)
        hbm, hbm_src = hbm_peak()
        roofline = {"bound": "hbm", "achieved": nbytes / sm_s / 1e9, "peak": hbm, "unit": "GB/s",
                    "frac": nbytes / sm_s / 1e9 / hbm, "traffic": None, "peak_source": hbm_src,
                    "kernel": "fa_std::softmax_rows_kernel", "algorithmic_bytes": nbytes,
                    "step_tflops": achieved}
    launches = int(sum_over_ranks(args.steps * launches_per_step, dist, dev))
    srt = sorted(launch_ms)
    step_ms = {"min": srt[0], "median": srt[len(srt) // 2], "max": srt[-1],
               "first5_mean": sum(launch_ms[:5]) / min(5, len(launch_ms)),
               "launches": len(launch_ms), "note": "single launches after the timed region"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and bwd is None:
        cpu = cpu_baseline(w, w.seed)

    # the other configurations of the target, on one GPU only (a multi-GPU
    # run reports the headline problem alone)
    per_config = None
    if world == 1 and not args.no_per_config and args.path == "fused" and w.name == DEFAULT_WORKLOAD:
        per_config = {}
        for name, path in EXTRA_CONFIGS:
            key = name if path == "forward" else f"{name}_backward"
            per_config[key] = measure_config(name, path, dev)

    if dist is not None:
        dist.barrier()
    if rank == 0:
        in_bytes = 4 * q.numel() * q.element_size() + lse.numel() * 4
        line = {
            "metric": METRIC if bwd is None else METRIC.replace("attention fwd", "attention bwd"),
            "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * elapsed_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16 Q/K/V per rank)",
            "config": {**w.as_config(), "parallelism": f"replicas{world}", "path": args.path,
                       **({"num_splits": splits} if splits is not None else {}),
                       "l2": (f"inputs+outputs {in_bytes / 1e6:.0f} MB > L2 126 MB, no flush"
                              if in_bytes > L2_BYTES else "L2 not flushed (inputs < L2)")},
            "pct_of_peak": 100.0 * value / world / peak,
            "roofline": roofline,
            "e2e": {"value": weak_scaling_value(flops, world, e2e_steps, e2e_s), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches,
            "step_ms": step_ms,
            "clocks": clocks,
            "cpu_baseline": cpu,
            **({"per_config": per_config} if per_config is not None else {}),
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------------------
# experiments (one GPU): exact vs block-sparse at matched output error
# ---------------------------------------------------------------------------

def retained_pairs(layout, N: int, causal: bool, bq: int, bk: int) -> int:
    """Allowed (query, key) pairs a block layout keeps, causal mask included."""
    import numpy as np

    total = 0
    for r, row in enumerate(layout):
        q_lo, q_hi = r * bq, min(N, (r + 1) * bq)  # rows [q_lo, q_hi)
        for c, keep in enumerate(row):
            if not keep:
                continue
            k_lo, k_hi = c * bk, min(N, (c + 1) * bk)  # keys [k_lo, k_hi)
            if not causal:
                total += (q_hi - q_lo) * (k_hi - k_lo)
                continue
            i = np.arange(q_lo, q_hi)  # keys j <= i
            total += int(np.clip(i + 1 - k_lo, 0, k_hi - k_lo).sum())
    return total


def time_launches(fn, steps: int, warmup: int, stream) -> float:
    """Average milliseconds per call of ``fn`` (CUDA events on ``stream``)."""
    import torch

    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def fp32_reference_rows(q, k, v, scale: float, causal: bool, rows):
    """Plain PyTorch fp32 attention for sampled rows [R, 3] of (b, h, i), on the GPU."""
    import torch

    out = torch.empty((rows.shape[0], q.shape[-1]), dtype=torch.float32, device=q.device)
    keys = torch.arange(q.shape[2], device=q.device)
    for bh in torch.unique(rows[:, 0] * q.shape[1] + rows[:, 1]).tolist():
        b, h = divmod(bh, q.shape[1])
        sel = ((rows[:, 0] == b) & (rows[:, 1] == h)).nonzero()[:, 0]
        i = rows[sel, 2].to(q.device)
        s = (q[b, h, i].float() @ k[b, h].float().T) * scale
        if causal:
            s = s.masked_fill(keys[None, :] > i[:, None], float("-inf"))
        out[sel.to(q.device)] = torch.softmax(s, dim=-1) @ v[b, h].float()
    return out


def run_sparse_experiment(args, w):
    """Exact fused attention vs block-sparse bands of growing width.

    Three input families of the workload's shape: ``local`` and
    ``local_sharp`` (make_local_qkv with a positional score of 10 and 20 at
    distance 0: scores fall off with the query-key distance) and ``iid``
    (N(0, 1), no structure).  For each band width the block-sparse kernel is timed and its
    output error is measured, on sampled rows, against a plain fp32 PyTorch
    reference of exact attention; the exact kernel's own error is measured the
    same way.  One JSON line per point, then one summary line per family with
    the narrowest band that matches (a) the parity tolerance (max 2e-2, mean
    2e-3) and (b) the exact kernel's own error (max and mean within 2x).
    """
    import numpy as np
    import torch

    from exact_softmax_attention_02_b200 import fa
    from exact_softmax_attention_02_b200.inputs import (local_block_layout, make_local_qkv, make_qkv,
                                                        sample_rows)

    if not torch.cuda.is_available():
        raise SystemExit("the experiment needs a CUDA device")
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    steps, warmup = max(3, min(args.steps, 20)), args.warmup
    rows = sample_rows(w.B, w.H, w.N, 2048, w.seed)
    n_kb = -(-w.N // fa.BLOCK_K)
    widths = [x for x in (0, 128, 256, 512, 1024, 2048, 4096, 8192, 16384, 32768) if x < w.N]
    allowed = retained_pairs([[True] * n_kb] * (-(-w.N // fa.BLOCK_Q)), w.N, w.causal,
                             fa.BLOCK_Q, fa.BLOCK_K)
    for family in ("local", "local_sharp", "iid"):
        if family.startswith("local"):
            q_h, k_h, v_h = make_local_qkv(w.B, w.H, w.N, w.d, w.seed,
                                           peak=10.0 if family == "local" else 20.0)
        else:
            q_h, k_h, v_h = make_qkv(w.B, w.H, w.N, w.d, w.seed)
        q, k, v = (t.to(dev) for t in (q_h, k_h, v_h))
        ref = fp32_reference_rows(q, k, v, w.scale, w.causal, rows)
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)

        def err(out):
            got = out[rows[:, 0], rows[:, 1], rows[:, 2]].float()
            e = (got - ref).abs()
            return float(e.max()), float(e.mean())

        ms_exact = time_launches(lambda: fa.fa_fwd(q, k, v, o, lse, scale=w.scale, causal=w.causal,
                                                   stream=stream), steps, warmup, stream)
        o_exact = o.clone()
        ex_max, ex_mean = err(o_exact)
        base = {"experiment": "exact_vs_block_sparse", "workload": w.name, "inputs": family}
        print(json.dumps({**base, "kernel": "exact", "density": 1.0, "ms": ms_exact,
                          "tflops": w.flops / ms_exact / 1e9, "err_max": ex_max, "err_mean": ex_mean}),
              flush=True)
        points = []
        for width in widths:
            for sinks in (0, 1):
                lay = local_block_layout(w.N, width, w.causal, fa.BLOCK_Q, fa.BLOCK_K, sinks=sinks)
                rp, ci = fa.block_layout_to_csr(lay, device=dev)
                density = retained_pairs(lay, w.N, w.causal, fa.BLOCK_Q, fa.BLOCK_K) / allowed
                ms = time_launches(lambda: fa.fa_fwd_block_sparse(q, k, v, o, rp, ci, lse, scale=w.scale,
                                                                  causal=w.causal, stream=stream),
                                   steps, warmup, stream)
                if fa.device_status(stream) != 0:
                    raise RuntimeError("block-sparse kernel reported a device failure")
                e_max, e_mean = err(o)
                d_exact = float((o.float() - o_exact.float()).abs().max())
                pt = {**base, "kernel": "block_sparse", "window": width, "sinks": sinks,
                      "density": density, "ms": ms, "speedup_vs_exact": ms_exact / ms,
                      "tflops_retained": w.flops * density / ms / 1e9,
                      "err_max": e_max, "err_mean": e_mean, "max_diff_vs_exact_kernel": d_exact}
                points.append(pt)
                print(json.dumps(pt), flush=True)

        def narrowest(ok):
            good = [p for p in points if ok(p)]
            return min(good, key=lambda p: p["ms"]) if good else None

        tol = narrowest(lambda p: p["err_max"] <= 2e-2 and p["err_mean"] <= 2e-3)
        own = narrowest(lambda p: p["err_max"] <= 2 * ex_max and p["err_mean"] <= 2 * ex_mean)
        summ = {**base, "summary": True, "exact_ms": ms_exact, "exact_err_max": ex_max,
                "exact_err_mean": ex_mean}
        for key, p in (("at_parity_tolerance", tol), ("at_exact_kernel_error", own)):
            summ[key] = None if p is None else {x: p[x] for x in ("window", "sinks", "density", "ms",
                                                                  "speedup_vs_exact", "err_max", "err_mean")}
        print(json.dumps(summ), flush=True)
        del q, k, v, o, lse, o_exact
    return 0


def run_tile_experiment(args, w):
    """Wall-clock time of the fused forward against tile size and head width.

    Tile shapes: 256 or 128 query rows per CTA (two 128-row tiles that
    ping-pong, or one; the query tile is the tensor core's 128 rows) times 128
    or 64 keys per score tile.  Head widths 64 and 128, sequence lengths 1K to
    64K with the token count B*H*N fixed at 2^19 (so every point holds the same
    inputs), both masks.  One JSON line per point (CUDA-event time per launch,
    TFLOP/s), then one line per (d, N, mask) naming the fastest shape.  Inputs
    are N(0, 1), seeded.
    """
    import torch

    from exact_softmax_attention_02_b200 import fa
    from exact_softmax_attention_02_b200.inputs import make_qkv

    if not torch.cuda.is_available():
        raise SystemExit("the experiment needs a CUDA device")
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    steps, warmup = max(3, min(args.steps, 20)), args.warmup
    tokens = 1 << 19
    peak, peak_src = tensor_peak()
    shapes = [(256, 128), (256, 64), (128, 128), (128, 64)]  # (query rows per CTA, keys per tile)
    for d in (64, 128):
        for N in (1024, 4096, 16384, 65536):
            H = tokens // N
            q_h, k_h, v_h = make_qkv(1, H, N, d, seed=N + d)
            q, k, v = (t.to(dev) for t in (q_h, k_h, v_h))
            o = torch.empty_like(q)
            lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
            for causal in (False, True):
                flops = 4.0 * H * N * N * d / (2 if causal else 1)
                best = None
                for query_rows, key_tile in shapes:
                    ms = time_launches(lambda: fa.fa_fwd_tile_config(q, k, v, o, lse, query_rows=query_rows,
                                                                     key_tile=key_tile, causal=causal,
                                                                     stream=stream),
                                       steps, warmup, stream)
                    if fa.device_status(stream) != 0:
                        raise RuntimeError("kernel reported a device failure")
                    tf = flops / ms / 1e9
                    pt = {"experiment": "tile_sweep", "B": 1, "H": H, "N": N, "d": d, "causal": causal,
                          "query_tile": 128, "query_rows_per_cta": query_rows, "key_tile": key_tile,
                          "ms": ms, "tflops": tf, "pct_of_peak": 100.0 * tf / peak, "peak_source": peak_src}
                    print(json.dumps(pt), flush=True)
                    if best is None or ms < best[2]:
                        best = (query_rows, key_tile, ms)
                print(json.dumps({"experiment": "tile_sweep", "summary": True, "N": N, "d": d,
                                  "causal": causal, "best_query_rows_per_cta": best[0],
                                  "best_key_tile": best[1]}), flush=True)
            del q, k, v, o, lse
    return 0


def main(argv=None):
    from exact_softmax_attention_02_b200.inputs import WORKLOADS

    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--path", default="fused", choices=["fused", "splitkv", "standard", "backward"],
                    help="fused: fa_fwd; splitkv: fa_fwd_splitkv (key ranges + merge); "
                         "standard: the materialising comparator (GEMM, softmax, GEMM); "
                         "backward: fa_bwd (dQ, dK, dV)")
    ap.add_argument("--splits", type=int, default=0, help="splitkv: key ranges (0 = default)")
    ap.add_argument("--experiment", default=None, choices=["sparse", "tiles"],
                    help="sparse: exact vs block-sparse bands at matched output error; tiles: "
                         "time against key-tile width and head width (1 GPU, JSON lines; not a "
                         "bench line)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the other configurations (d=64, long-context causal, backward) "
                         "measured after the headline problem")
    ap.add_argument("--ref-step-seconds", type=float, default=8.0,
                    help="reference arm: target oracle seconds per step (bounded sample)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.steps < 1:
        ap.error("--steps must be >= 1")
    w = WORKLOADS[args.workload]
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # not under torchrun: start one process per GPU the same way the
        # harness does, on the loopback address
        cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
               f"--nproc-per-node={args.gpus}", "--master-addr=127.0.0.1",
               "--master-port=29517", os.path.abspath(__file__), *(argv or sys.argv[1:])]
        return subprocess.call(cmd)
    if args.impl == "reference":
        return run_reference(args, w)
    if args.experiment == "sparse":
        return run_sparse_experiment(args, w)
    if args.experiment == "tiles":
        return run_tile_experiment(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
