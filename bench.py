#!/usr/bin/env python
"""Throughput of the clip-parallel temporal modules (Video-Infinity) on B200.

One step = one pass of the whole hot path over one latent video: dual-domain
attention (q, k, v -> out), the clip-padded temporal conv (x -> y) and the
global-statistics GroupNorm (x' -> z), each through the C ABI of libvi.
Inputs are seeded synthetic tensors of the workload's shape (the pages'
512x320 video at a /8 latent, F = 1024 frames in 64 clips by default), already
resident in HBM when the timed region starts; every tensor (1.68 GB) is larger
than L2, so no flush is needed between steps.

Metric: temporal-module tokens/s, tokens = F * P (= F * H'W') per step, for
the whole job (all ranks).  With --gpus N every rank runs its own video
(weak scaling; the path has no exchange between independent videos).

Printed (rank 0, one JSON line): value, ms_per_step, a per-kernel breakdown,
the roofline of the dominant kernel (algorithmic bytes or flops over its
CUDA-event time, against MEASURED_PEAKS.json), the oracle timed on the host
cores as cpu_baseline, an end-to-end figure through host buffers (e2e), the
SM clocks sampled during the timed region, and the number of libvi kernel
launches in the timed region.

--impl reference times the fp64 CPU oracle itself on a bounded sample of the
same workload (the only reference this method has: the pages ship no code).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "bf16_F1024_P2560_C320"
# Nominal per-GPU figures (B200 HGX: HBM3e 7.7 TB/s, dense bf16 2.25 PFLOP/s), reported
# beside the measured denominators for context.
NOMINAL = {"hbm_gbs": 7700.0, "bf16_tflops": 2250.0}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--e2e-chunks", type=int, default=16,
                    help="position chunks of the end-to-end pipeline")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-second-workload", action="store_true",
                    help="skip the per-kernel figures of the other F=1024 workload")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle sample")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------
# distributed plumbing


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(backend: str):
    import torch.distributed as dist
    world, rank, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        from datetime import timedelta
        dist.init_process_group(backend, timeout=timedelta(seconds=120))
    return world, rank


def max_over_ranks(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------------------
# accounting


def kernel_work(w):
    """Algorithmic bytes (attention, GroupNorm) and flops (conv) per step.

    attention: read q, k, v and write out once: 4 S bytes (halo and global
               frames are re-reads that must come from L2, not HBM).
    GroupNorm: one read for the statistics, one read and one write to
               normalise: 3 S bytes.
    conv:      2 * k * C^2 flops per token (a C x kC contraction); bytes
               2 S + weights.
    """
    S = w.P * w.F * w.C * w.elem_bytes
    return {
        "dual_attn": {"bytes": 4 * S},
        "temporal_conv": {"flops": 2 * w.k * w.C * w.C * w.tokens,
                          "bytes": 2 * S + w.C * w.C * w.k * w.elem_bytes},
        "groupnorm_global": {"bytes": 3 * S},
    }


def choose_tensor_peak(peaks, timed_s: float, clk) -> tuple[float, str]:
    """The measured bf16 peak that fits the timed region: the burst figure,
    unless the region lasts seconds and its SM clock sits well below the
    maximum (the power-capped regime the sustained figure was measured in)."""
    burst = peaks.get("bf16_tflops")
    sustained = peaks.get("bf16_tflops_sustained", burst)
    mhz, max_mhz = clk.get("sm_mhz"), clk.get("sm_max_mhz")
    long_capped = timed_s >= 2.0 and mhz and max_mhz and mhz < 0.85 * max_mhz
    return (sustained, "bf16_tflops_sustained") if long_capped else (burst, "bf16_tflops")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.02):
        self.index, self.period = index, period_s
        self.samples, self.mem_samples, self.reasons = [], [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            return self
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.mem_samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_MEM))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for b, name in self.REASONS.items():
                    if bits & b and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread:
            self._thread.join(timeout=1.0)
        return False

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"],
                    "samples": 0}
        out = {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
               "reasons": sorted(self.reasons), "samples": len(self.samples)}
        if self.mem_samples:
            out["mem_mhz"] = statistics.median(self.mem_samples)
        return out


def clock_anomaly(clk) -> str | None:
    """Why a timed region's clock record disqualifies it, or None."""
    bad = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"} & set(clk["reasons"])
    if bad:
        return "throttle: " + ",".join(sorted(bad))
    if clk["sm_mhz"] and clk["sm_max_mhz"] and clk["sm_mhz"] < 0.9 * clk["sm_max_mhz"] \
            and "sw_power_cap" not in clk["reasons"]:
        return f"sm clock {clk['sm_mhz']} of {clk['sm_max_mhz']} MHz with no reason"
    return None


# ---------------------------------------------------------------------------
# inputs


def host_inputs(w, pinned: bool):
    """Seeded synthetic inputs of workload w as torch CPU tensors (bf16 or fp32)."""
    import torch

    import synth
    out = {}
    for name in ("q", "k", "v", "conv_x", "conv_w", "conv_b", "gn_x", "gn_gamma", "gn_beta"):
        a = synth.make(w, name)
        t = torch.from_numpy(a)
        if w.dtype == "bf16":
            t = t.view(torch.bfloat16)
        out[name] = t.pin_memory() if pinned else t
    return out


INPUT_NAMES = ("q", "k", "v", "conv_x", "conv_w", "conv_b", "gn_x", "gn_gamma", "gn_beta")


def shared_host_inputs(w, rank: int, world: int, pinned: bool, device=None):
    """Every rank's copy of the seeded inputs of workload w.

    With one rank this is host_inputs().  With several, rank 0 generates them
    once and broadcasts each tensor (through `device` for NCCL, on the host for
    gloo): every replica gets the same video without each rank repeating the
    generation on the shared host cores.  A setup step, outside any timed region."""
    import torch
    import torch.distributed as dist

    if world == 1 or not dist.is_initialized():
        return host_inputs(w, pinned)
    import synth
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    src = host_inputs(w, pinned) if rank == 0 else None
    out = {}
    for name in INPUT_NAMES:
        shape = synth.shape_of(w, name)
        t = src[name] if rank == 0 else torch.empty(shape, dtype=dt)
        if device is not None:
            d = t.to(device) if rank == 0 else torch.empty(shape, dtype=dt, device=device)
            dist.broadcast(d, src=0)
            t = d.cpu() if rank != 0 else t
        else:
            dist.broadcast(t, src=0)
        out[name] = t.pin_memory() if pinned and not t.is_pinned() else t
    return out


# ---------------------------------------------------------------------------
# our arm


def run_ours(args):
    import torch

    import clip_temporal_modules_b200 as vi
    import synth

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist("nccl")
    w = synth.BY_NAME[args.workload]
    stream = torch.cuda.current_stream()

    host = shared_host_inputs(w, rank, world, pinned=True, device=dev)
    d = {k: v.to(dev, non_blocking=True) for k, v in host.items()}
    out = torch.empty_like(d["q"])
    y = torch.empty_like(d["conv_x"])
    z = torch.empty_like(d["gn_x"])
    torch.cuda.synchronize()

    names = ("dual_attn", "temporal_conv", "groupnorm_global")

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        vi.dual_attn(d["q"], d["k"], d["v"], out, N=w.N, heads=w.heads, n_pre=w.n_pre,
                     n_post=w.n_post, n_global=w.n_global)
        if ev is not None:
            ev[1].record(stream)
        vi.temporal_conv(d["conv_x"], d["conv_w"], d["conv_b"], y, N=w.N)
        if ev is not None:
            ev[2].record(stream)
        vi.groupnorm_global(d["gn_x"], d["gn_gamma"], d["gn_beta"], z, N=w.N, groups=w.groups,
                            eps=w.eps)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    vi.take_device_errors()

    def timed():
        """The timed region: K steps between a barrier + synchronize on each side."""
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)]
               for _ in range(args.steps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(dev)
        torch.cuda.synchronize()
        launches0 = vi.launch_count()
        with ClockSampler(dev.index) as clocks:
            t0.record(stream)
            for i in range(args.steps):
                step(evs[i])
            t1.record(stream)
            torch.cuda.synchronize()
        launches = vi.launch_count() - launches0
        barrier(dev)
        elapsed_ms = max_over_ranks(t0.elapsed_time(t1), dev)
        vi.take_device_errors()
        per_kernel = {n: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs)
                      for j, n in enumerate(names)}
        return elapsed_ms, per_kernel, launches, clocks.summary()

    elapsed_ms, per_kernel, launches, clk = timed()
    remeasured = None
    # A run that saw a hardware or thermal slowdown, or SM clocks well below
    # their maximum with no reason given, is measured once more (every rank
    # takes the same decision, since the timed region holds collectives).
    bad = clock_anomaly(clk)
    if max_over_ranks(1.0 if bad else 0.0, dev) > 0:
        remeasured = {"first_ms_per_step": round(elapsed_ms / args.steps, 4), "first_clocks": clk,
                      "why": bad or "another rank"}
        elapsed_ms, per_kernel, launches, clk = timed()
    ms_per_step = elapsed_ms / args.steps
    tokens = w.tokens * world * args.steps
    value = tokens / (elapsed_ms / 1e3)

    peaks, peak_src = load_peaks()
    tensor_peak, tensor_key = choose_tensor_peak(peaks, elapsed_ms / 1e3, clk)
    kernels = kernel_figures(w, per_kernel, peaks, tensor_peak)
    dom = max(names, key=lambda n: per_kernel[n])
    kd = kernels[dom]
    traffic = load_traffic(dom, w)
    roofline = {"kernel": dom, "bound": kd["bound"], "achieved": kd["achieved"],
                "peak": tensor_peak if kd["bound"] == "tensor" else peaks["hbm_gbs"],
                "unit": kd["unit"], "frac": kd["frac"], "traffic": traffic,
                "peak_source": f"{peak_src} ({tensor_key if kd['bound'] == 'tensor' else 'hbm_gbs'})"}
    if kd["bound"] == "tensor":
        # Both measured bf16 figures, whichever the timed region calls for.
        roofline["frac_burst"] = round(kd["achieved"] / peaks["bf16_tflops"], 4)
        roofline["frac_sustained"] = round(
            kd["achieved"] / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]), 4)
    nom = NOMINAL["bf16_tflops"] if kd["bound"] == "tensor" else NOMINAL["hbm_gbs"]
    roofline["nominal"] = {"peak": nom, "frac": round(kd["achieved"] / nom, 4)}

    result = {
        "metric": "temporal-module tokens/s (F*H'W') at F=1024",
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (seeded SplitMix64 + Box-Muller; q/k/v/x N(0,1), conv w N(0,1/(kC)), GN x N(0.5,2))",
        "config": {"workload": w.name, "F": w.F, "N_clips": w.N, "P": w.P, "C": w.C,
                   "heads": w.heads, "d": w.d, "n_pre": w.n_pre, "n_post": w.n_post,
                   "n_global": w.n_global, "k": w.k, "groups": w.groups,
                   "tokens_per_step_per_gpu": w.tokens,
                   "parallelism": f"replica x{world} (one video per GPU)",
                   "l2": "no flush: every tensor (%.2f GB) exceeds L2" % (w.act_bytes / 1e9)},
        "kernels": kernels,
        "roofline": roofline,
        "gpu_launches": int(launches),
        "clocks": clk,
    }

    if remeasured is not None:
        result["remeasured"] = remeasured
    # The attention module first among the extra blocks, after a short idle:
    # it then starts from the state the headline region started from (the
    # blocks after it, the CUDA-core attention path above all, keep the GPU at
    # its power cap for a good part of a second).  Each block carries its own
    # clock record.
    time.sleep(0.5)
    result["temporal_attention_module"] = attention_module(w, d, out, y, z, stream)
    result["attn_ablations"] = attn_ablations(w, d, out, y, z, stream)
    result["attn_generic_path"] = attn_generic_path(w, d, out, stream)
    result["attn_halo16"] = attn_halo16(w, d, out, stream)
    result["groupnorm_conv_fused"] = fused_gn_conv(w, d, y, z, stream)
    if w.dtype == "bf16" and w.F % 8 == 0 and w.N % 8 == 0:
        try:
            result["clip_parallel_emulated"] = clip_parallel_emulated(w, d, stream)
        except Exception as e:       # an extra figure: never lose the headline line over it
            result["clip_parallel_emulated"] = {"error": f"{type(e).__name__}: {e}"[:300]}

    other = "bf16_F1024_P640_C640" if w.name == DEFAULT_WORKLOAD else None
    if other and not args.no_second_workload:
        try:
            result["kernels_" + other] = second_workload(other, dev, stream)
        except Exception as e:       # an extra figure: never lose the headline line over it
            result["kernels_" + other] = {"error": f"{type(e).__name__}: {e}"[:300]}

    if not args.no_e2e:
        result["e2e"] = run_e2e(args, w, host, dev, stream)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)

    if rank == 0:
        print(json.dumps(result), flush=True)
    cleanup()


def kernel_figures(w, per_kernel, peaks, tensor_peak):
    """Per-kernel ms, achieved rate and fraction of the measured peak."""
    work = kernel_work(w)
    kernels = {}
    for n, ms in per_kernel.items():
        if "flops" in work[n]:
            ach = work[n]["flops"] / (ms / 1e3) / 1e12
            kernels[n] = {"ms": round(ms, 4), "achieved": round(ach, 1), "unit": "TFLOP/s",
                          "frac": round(ach / tensor_peak, 4), "bound": "tensor",
                          "tokens_per_s": round(w.tokens / (ms / 1e3), 1)}
        else:
            ach = work[n]["bytes"] / (ms / 1e3) / 1e9
            kernels[n] = {"ms": round(ms, 4), "achieved": round(ach, 1), "unit": "GB/s",
                          "frac": round(ach / peaks["hbm_gbs"], 4), "bound": "hbm",
                          "tokens_per_s": round(w.tokens / (ms / 1e3), 1)}
    return kernels


def second_workload(name, dev, stream, steps=20, warmup=5):
    """The three kernels on another F=1024 workload (its own seeded inputs,
    timed after the headline region like the other extras): per-kernel time
    and fraction of the measured peaks, with the clocks of its timed steps."""
    import torch

    import clip_temporal_modules_b200 as vi
    import synth
    w = synth.BY_NAME[name]
    host = host_inputs(w, pinned=False)
    d = {k: v.to(dev) for k, v in host.items()}
    del host
    out, y, z = (torch.empty_like(d["q"]) for _ in range(3))
    names = ("dual_attn", "temporal_conv", "groupnorm_global")

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        vi.dual_attn(d["q"], d["k"], d["v"], out, N=w.N, heads=w.heads, n_pre=w.n_pre,
                     n_post=w.n_post, n_global=w.n_global)
        if ev is not None:
            ev[1].record(stream)
        vi.temporal_conv(d["conv_x"], d["conv_w"], d["conv_b"], y, N=w.N)
        if ev is not None:
            ev[2].record(stream)
        vi.groupnorm_global(d["gn_x"], d["gn_gamma"], d["gn_beta"], z, N=w.N, groups=w.groups,
                            eps=w.eps)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clocks:
        t0.record(stream)
        for i in range(steps):
            step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize()
    vi.take_device_errors()
    per_kernel = {n: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs)
                  for j, n in enumerate(names)}
    total_ms = t0.elapsed_time(t1)
    clk = clocks.summary()
    peaks, _ = load_peaks()
    tensor_peak, tensor_key = choose_tensor_peak(peaks, total_ms / 1e3, clk)
    res = {"workload": w.name, "steps": steps, "ms_per_step": round(total_ms / steps, 4),
           "tokens_per_s": round(w.tokens * steps / (total_ms / 1e3), 1),
           "kernels": kernel_figures(w, per_kernel, peaks, tensor_peak),
           "tensor_peak": f"{tensor_key} ({tensor_peak})", "clocks": clk}
    del d, out, y, z
    torch.cuda.empty_cache()
    return res


def attn_ablations(w, d, out, y, z, stream, reps=10):
    """Dual attention under the write-up's ablation settings (timed after the
    headline region): no global context, no local context, no exchange.

    Timed the way the headline splits its step: each attention call between
    its own pair of events, inside the step's order (attention, conv,
    GroupNorm), so that its predecessor and the L2 state it meets match the
    headline's; "full_8_8_16" repeats the headline's own setting as a check,
    and the block carries its own clock record."""
    import clip_temporal_modules_b200 as vi
    S = w.P * w.F * w.C * w.elem_bytes
    res = {}

    def rest():
        vi.temporal_conv(d["conv_x"], d["conv_w"], d["conv_b"], y, N=w.N)
        vi.groupnorm_global(d["gn_x"], d["gn_gamma"], d["gn_beta"], z, N=w.N, groups=w.groups,
                            eps=w.eps)

    settings = {"full_8_8_16": (w.n_pre, w.n_post, w.n_global), "local_only_8_8_0": (8, 8, 0),
                "global_only_0_0_16": (0, 0, 16), "no_sync_0_0_0": (0, 0, 0)}
    dev = d["q"].device
    with ClockSampler(dev.index) as clocks:
        for name, (a, b_, g) in settings.items():
            res[name] = _ablation(w, d, out, rest, stream, reps, S, a, b_, g)
    res["clocks"] = clocks.summary()
    return res


def attn_generic_path(w, d, out, stream, reps=2):
    """The same attention with n_global = 32, outside the tensor-core fast
    path (which takes d = 64, n_global <= 16, and clips of 16 frames with
    n_pre, n_post <= 16 or of 8 with n_pre, n_post <= 8):
    one warp per query frame on CUDA cores.  Reported so that the cost off
    the fast path is visible, not as a tuned figure."""
    import torch

    import clip_temporal_modules_b200 as vi
    n_pre, n_post, n_global = w.n_pre, w.n_post, min(32, w.F)

    def attn():
        vi.dual_attn(d["q"], d["k"], d["v"], out, N=w.N, heads=w.heads, n_pre=n_pre,
                     n_post=n_post, n_global=n_global)
    attn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        attn()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    S = w.P * w.F * w.C * w.elem_bytes
    return {"n_pre": n_pre, "n_post": n_post, "n_global": n_global, "ms": round(ms, 4),
            "GB/s": round(4 * S / (ms / 1e3) / 1e9, 1), "path": "dual_attn_generic_staged (CUDA cores, key lists staged in shared memory)"}


def attn_halo16(w, d, out, stream, reps=10):
    """The attention with n_pre = n_post = 16 (a whole clip of context on each
    side): the tensor-core kernel with its 16-row windows."""
    import torch

    import clip_temporal_modules_b200 as vi
    n = min(16, w.F // w.N)

    def attn():
        vi.dual_attn(d["q"], d["k"], d["v"], out, N=w.N, heads=w.heads, n_pre=n, n_post=n,
                     n_global=w.n_global)
    for _ in range(2):
        attn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        attn()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    S = w.P * w.F * w.C * w.elem_bytes
    return {"n_pre": n, "n_post": n, "n_global": w.n_global, "ms": round(ms, 4),
            "GB/s": round(4 * S / (ms / 1e3) / 1e9, 1)}


def _ablation(w, d, out, rest, stream, reps, S, a, b_, g):
    """One ablation setting, timed per call inside the step order."""
    import torch

    import clip_temporal_modules_b200 as vi

    def attn():
        vi.dual_attn(d["q"], d["k"], d["v"], out, N=w.N, heads=w.heads, n_pre=a, n_post=b_,
                     n_global=g)
    for _ in range(2):
        attn()
        rest()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(reps)]
    for e0, e1 in evs:
        e0.record(stream)
        attn()
        e1.record(stream)
        rest()
    torch.cuda.synchronize()
    ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in evs)
    return {"ms": round(ms, 4), "GB/s": round(4 * S / (ms / 1e3) / 1e9, 1)}


def fused_gn_conv(w, d, y, z, stream, reps=10):
    """GroupNorm -> conv of one tensor: the fused call against the two calls
    (timed after the headline region)."""
    import torch

    import clip_temporal_modules_b200 as vi

    def two():
        vi.groupnorm_global(d["gn_x"], d["gn_gamma"], d["gn_beta"], z, N=w.N, groups=w.groups,
                            eps=w.eps)
        vi.temporal_conv(z, d["conv_w"], d["conv_b"], y, N=w.N)

    def fused():
        vi.groupnorm_conv(d["gn_x"], d["gn_gamma"], d["gn_beta"], d["conv_w"], d["conv_b"], y,
                          N=w.N, groups=w.groups, eps=w.eps)

    res = {}
    for name, fn in (("two_calls", two), ("fused", fused)):
        for _ in range(2):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        res[name] = {"ms": round(ms, 4), "tokens_per_s": round(w.tokens / (ms / 1e3), 1)}
    return res


def attention_module(w, d, out, y, z, stream, reps=3):
    """Temporal attention module (q/k/v projections, dual attention, output
    projection) on the workload's input, timed after the headline region."""
    import torch

    import clip_temporal_modules_b200 as vi
    import synth
    dev = out.device
    mk = lambda t: torch.from_numpy(synth.make(w, t)).view(torch.bfloat16).to(dev)
    wq, bq, wo, bo = (mk(t) for t in ("w_qkv", "b_qkv", "w_out", "b_out"))
    n = int(vi.lib().vi_temporal_attention_workspace_bytes(w.F, w.P, w.C))
    ws = torch.empty(n // 2, dtype=torch.bfloat16, device=dev)
    x = d["conv_x"]

    from clip_temporal_modules_b200._binding import temporal_attention_forced_form

    def run():
        vi.temporal_attention(x, wq, bq, wo, bo, y, ws, N=w.N, heads=w.heads, n_pre=w.n_pre,
                              n_post=w.n_post, n_global=w.n_global)

    def run_unfused():
        temporal_attention_forced_form(x, wq, bq, wo, bo, y, ws, N=w.N, heads=w.heads,
                                       fused=False, n_pre=w.n_pre, n_post=w.n_post,
                                       n_global=w.n_global)

    def timed(fn):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    from clip_temporal_modules_b200._binding import dual_attn_oproj

    def run_kernel():    # the fused attention + output projection kernel alone
        dual_attn_oproj(d["q"], d["k"], d["v"], wo, bo, y, N=w.N, heads=w.heads, n_pre=w.n_pre,
                        n_post=w.n_post, n_global=w.n_global)

    for _ in range(2):
        run()
        run_unfused()
        run_kernel()
    # Three interleaved rounds of each; the median round of each.  The clock is
    # sampled every 5 ms per round: the module draws enough power that the
    # power cap can lower the clock within a few tens of milliseconds.
    fused, unfused, kern, round_clocks = [], [], [], []
    idx = dev.index if dev.index is not None else 0
    with ClockSampler(idx) as clocks:
        for _ in range(3):
            with ClockSampler(idx, period_s=0.005) as rc:
                fused.append(timed(run))
                unfused.append(timed(run_unfused))
                kern.append(timed(run_kernel))
            round_clocks.append(rc.summary())
    ms, ms_unfused, ms_kern = sorted(fused)[1], sorted(unfused)[1], sorted(kern)[1]
    del ws
    flops = 4 * 2 * w.C * w.C * w.tokens
    S = w.tokens * w.C * 2
    # x read, q/k/v written and read back, out written (a stays on chip when
    # the output projection is fused into the attention)
    hbm = 8 * S
    return {"ms": round(ms, 4), "tokens_per_s": round(w.tokens / (ms / 1e3), 1),
            "projection_tflops_total": round(flops / 1e12, 3),
            "algorithmic_gb": round(hbm / 1e9, 3),
            "attention_then_output_gemm_ms": round(ms_unfused, 4),
            "rounds_ms": [round(t, 4) for t in fused],
            # q, k, v read and out written once (W_out comes from L2)
            "attention_oproj_kernel": {"ms": round(ms_kern, 4),
                                       "GB/s": round(4 * S / (ms_kern / 1e3) / 1e9, 1)},
            "attention_then_output_gemm_rounds_ms": [round(t, 4) for t in unfused],
            "round_sm_mhz": [c.get("sm_mhz") for c in round_clocks],
            "round_reasons": [c.get("reasons") for c in round_clocks],
            "clocks": clocks.summary()}


def clip_parallel_emulated(w, d, stream, world=8, reps=5):
    """The per-shard kernels of clip parallelism (frames sharded over `world`
    GPUs), emulated on this GPU: each shard's halo-padded storage is filled
    from the whole tensors beforehand (what the exchange would deliver into
    it), then the shard calls of every shard run back to back and are timed,
    per module and in total.  The exchange itself (NCCL) is not part of this
    figure."""
    import torch

    from clip_temporal_modules_b200._binding import (dual_attn_shard, groupnorm_shard_apply,
                                                     groupnorm_shard_stats, temporal_conv_shard)
    from clip_temporal_modules_b200.clip_parallel import (ShardLayout, extended_from_full,
                                                          global_frame_index)
    lays = [ShardLayout(w.F, w.N, world, r) for r in range(world)]
    gidx = global_frame_index(w.F, w.n_global)
    kg, vg = d["k"][:, gidx].contiguous(), d["v"][:, gidx].contiguous()
    shards = []
    for lay in lays:
        f0, f1 = lay.f0, lay.f0 + lay.F_loc
        q = d["q"][:, f0:f1].contiguous()
        shards.append({"q": q, "k": extended_from_full(d["k"], f0, f1, 8),
                       "v": extended_from_full(d["v"], f0, f1, 8),
                       "x": extended_from_full(d["conv_x"], f0, f1, w.k // 2),
                       "g": d["gn_x"][:, f0:f1].contiguous(), "out": torch.empty_like(q),
                       "y": torch.empty_like(q), "z": torch.empty_like(q)})

    def attn():
        for lay, sh in zip(lays, shards):
            dual_attn_shard(sh["q"], sh["k"], sh["v"], kg, vg, sh["out"], N_loc=lay.N_loc,
                            clip0=lay.clip0, N=w.N, heads=w.heads, n_pre=w.n_pre,
                            n_post=w.n_post, n_global=w.n_global)

    def conv():
        for sh in shards:
            temporal_conv_shard(sh["x"], d["conv_w"], d["conv_b"], sh["y"])

    # Each shard's statistics land in its slot of the gathered [W][groups][2]
    # tensor (what the all-gather delivers on every GPU).
    stats = torch.empty((world, w.groups, 2), dtype=torch.float64, device=d["q"].device)

    def gn():
        for i, sh in enumerate(shards):
            groupnorm_shard_stats(sh["g"], groups=w.groups, out=stats[i])
        for sh in shards:
            groupnorm_shard_apply(sh["g"], stats, d["gn_gamma"], d["gn_beta"], sh["z"], eps=w.eps)

    res = {"world": world}
    total = 0.0
    for name, fn in (("dual_attn", attn), ("temporal_conv", conv), ("groupnorm_global", gn)):
        for _ in range(2):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        res[name + "_ms"] = round(ms, 4)
        total += ms
    del shards
    torch.cuda.empty_cache()
    res.update({"ms_all_shards": round(total, 4),
                "tokens_per_s": round(w.tokens / (total / 1e3), 1),
                "what": f"{world} frame shards' kernels on one GPU, halo-padded storage filled; "
                        "exchange not included"})
    return res


def run_e2e(args, w, host, dev, stream):
    """Same step from and to pinned host buffers, through the package's
    HostPipeline: copy-in, compute and copy-out streams over position chunks."""
    import torch

    import clip_temporal_modules_b200 as vi
    world, _, _ = dist_env()
    res = {k: torch.empty_like(host["q"]).pin_memory() for k in ("out", "y", "z")}
    shape = vi.StepShape(F=w.F, N=w.N, P=w.P, C=w.C, heads=w.heads, n_pre=w.n_pre,
                         n_post=w.n_post, n_global=w.n_global, k=w.k, groups=w.groups, eps=w.eps)
    pipe = vi.HostPipeline(shape, dev, host["q"].dtype, chunks=args.e2e_chunks)

    pipe.run(host, res)
    torch.cuda.synchronize()
    barrier(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.e2e_steps):
        pipe.run(host, res)
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), dev)
    barrier(dev)
    del pipe
    return {"value": round(w.tokens * world * args.e2e_steps / (ms / 1e3), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": vi.HostPipeline.h2d_bytes(host),
            "d2h_bytes_per_step": vi.HostPipeline.d2h_bytes(res),
            "steps": args.e2e_steps, "ms_per_step": round(ms / args.e2e_steps, 3),
            "path": f"pinned host -> HostPipeline ({pipe_desc(args.e2e_chunks)}) -> libvi C ABI"
                    " -> pinned host"}


def pipe_desc(chunks: int) -> str:
    return f"copy-in / compute / copy-out streams, {chunks} position chunks"


def load_traffic(kernel, w):
    """DRAM bytes per launch from the committed ncu summary of this kernel.

    None when there is no capture for this workload, or when the kernel's
    sources have changed since the counters were taken (the summary records a
    hash of the source files it was measured with: the kernel's file and the
    headers it includes)."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as fh:
        d = json.load(fh)
    e = d.get(kernel, {}).get(w.name)
    if e is None:
        return None
    h = hashlib.sha256()
    for rel in e["sources"]:
        src = os.path.join(ROOT, "clip_temporal_modules_b200", rel)
        if not os.path.exists(src):
            return None
        with open(src, "rb") as fh:
            h.update(fh.read())
    if h.hexdigest()[:16] != e.get("sources_sha256_16"):
        return None
    return e.get("bytes_per_launch")


# ---------------------------------------------------------------------------
# the oracle on the host cores


def oracle_sample(w, positions: int):
    """One bounded sample of the workload: `positions` whole positions (all F frames,
    all C channels) through the three modules of the oracle.  GroupNorm takes its
    statistics over the sample (the same work per token as over the full tensor)."""
    import synth
    sub = w.with_(P=positions)
    return {name: synth.make(sub, name) for name in
            ("q", "k", "v", "conv_x", "conv_w", "conv_b", "gn_x", "gn_gamma", "gn_beta")}, sub


def oracle_step(inp, sub, nthreads: int = 0):
    """The three modules of the oracle on the sample (nthreads 0 = every host core)."""
    import oracle
    oracle.dual_attn(inp["q"], inp["k"], inp["v"], sub.F, sub.N, sub.heads, sub.d, sub.n_pre,
                     sub.n_post, sub.n_global, nthreads=nthreads)
    oracle.temporal_conv(inp["conv_x"], inp["conv_w"], inp["conv_b"], sub.F, sub.N, sub.k,
                         nthreads=nthreads)
    oracle.groupnorm_global(inp["gn_x"], inp["gn_gamma"], inp["gn_beta"], sub.F, sub.N,
                            sub.groups, sub.eps, nthreads=nthreads)


def calibrate_positions(w, seconds: float) -> int:
    inp, sub = oracle_sample(w, 1)
    t = time.perf_counter()
    oracle_step(inp, sub)
    per_pos = max(time.perf_counter() - t, 1e-3)
    return max(1, min(w.P, int(seconds / per_pos)))


def cpu_baseline(w, seconds: float):
    import oracle
    npos = calibrate_positions(w, seconds)
    inp, sub = oracle_sample(w, npos)
    t = time.perf_counter()
    oracle_step(inp, sub)
    dt = time.perf_counter() - t
    # The same oracle on one host thread, on a smaller sample (2 positions).
    inp1, sub1 = oracle_sample(w, min(2, w.P))
    t = time.perf_counter()
    oracle_step(inp1, sub1, nthreads=1)
    dt1 = time.perf_counter() - t
    return {"value": round(sub.tokens / dt, 1), "unit": "tokens/s", "cores": oracle.max_threads(),
            "kind": "oracle", "seconds": round(dt, 2),
            "sample": f"{npos} of {w.P} positions x all {w.F} frames x {w.C} channels of "
                      f"{w.name}, all three modules (GroupNorm statistics over the sample)",
            "single_thread": {"value": round(sub1.tokens / dt1, 1), "unit": "tokens/s",
                              "sample": f"{sub1.P} positions", "seconds": round(dt1, 2)}}


def run_reference(args):
    """The oracle, as it stands, on the host cores: each step is a bounded sample."""
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    import synth
    w = synth.BY_NAME[args.workload]
    budget = 120.0 / max(1, args.steps + args.warmup)        # whole run in ~2 minutes
    npos = calibrate_positions(w, min(budget, args.cpu_seconds))
    inp, sub = oracle_sample(w, npos)
    for _ in range(args.warmup):
        oracle_step(inp, sub)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(inp, sub)
    dt = time.perf_counter() - t
    value = sub.tokens * args.steps / dt
    cpu = {"value": round(value, 1), "unit": "tokens/s", "cores": oracle.max_threads(),
           "kind": "oracle",
           "sample": f"{npos} of {w.P} positions x all {w.F} frames x {w.C} channels of {w.name}"}
    print(json.dumps({
        "impl": "reference", "metric": "temporal-module tokens/s (F*H'W') at F=1024",
        "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)", "config": {"workload": w.name, "sample_positions": npos},
        "cpu_baseline": cpu,
        "e2e": {"value": round(value, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def cleanup():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        run_reference(args)
        return
    run_ours(args)


if __name__ == "__main__":
    main()
