#!/usr/bin/env python
"""Benchmark of the routed MoE FFN forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload mixtral]
    python bench.py --impl reference ...   # the fp64 CPU oracle, timed on host cores

One step = one moe_forward call over one batch of T tokens: router logits,
routing, scan, scatter, gate/up GEMM + SwiGLU, down GEMM + gate scaling,
combine. Weights and a ring of fresh x batches are resident in HBM before the
timed region; the expert weights (2.8 GB for the Mixtral-shaped layer) are
larger than L2, so no L2 flush is needed between steps. Every rank runs its
own replica on its own GPU ("replicas only": the layer has no exchange step);
the job value is the tokens of all ranks over the slowest rank's device time.
Ranks come from torchrun's environment, or, when none is set and --gpus N > 1,
from N processes this script spawns itself. Rank 0 prints one JSON line.

The default (Mixtral-shaped) run also times the weight-streaming decode shape
on the same weights: T = 32 tokens, 1000 back-to-back calls, each on its own
pre-generated x, reported under "decode" against the HBM bandwidth.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s and active TFLOP/s vs B200 bf16 roofline, Mixtral shape"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# (workload, weights) -> (DRAM bytes / algorithmic bytes of the gate/up kernel, the case the
# ratio was captured on), from one ncu capture of that kernel as built on a small case with
# the same rows per expert and kernel choice; absent = not captured for the current build.
# Algorithmic bytes are step_work's on the captured case (two experts).
_PREFILL_CASE = "T=1024 E=2 case (1024 rows per expert)"
_DECODE_CASE = "T=32 E=2 case"
_DSV3_CASE = "T=1024 E=32 d=7168 d_e=2048 k=8 +shared case (256 rows per expert)"
TRAFFIC_RATIO = {
    ("mixtral", "dtype"): (539.20 / 545.26, _PREFILL_CASE),
    ("deepseek_v3", "dtype"): (2199.70 / 2107.64, _DSV3_CASE),
    ("mixtral", "fp8"): (300.30 / 310.60, _PREFILL_CASE),
    ("decode", "fp8"): (240.30 / 237.46, _DECODE_CASE),
    ("decode", "mxfp4"): (131.30 / 127.43, _DECODE_CASE),
}
# the same for the down kernel
DOWN_TRAFFIC_RATIO = {
    ("mixtral", "dtype"): (343.40 / 310.38, _PREFILL_CASE),
    ("deepseek_v3", "dtype"): (1129.70 / 1138.75, _DSV3_CASE),
    ("mixtral", "fp8"): (220.10 / 192.97, _PREFILL_CASE),
    ("decode", "fp8"): (124.10 / 119.83, _DECODE_CASE),
    ("decode", "mxfp4"): (65.90 / 64.79, _DECODE_CASE),
}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mixtral",
                    choices=["mixtral", "deepseek_v3", "switch_zipf", "decode", "tiny_fp32",
                             "mixtral_profile", "decode_profile", "routing_profile",
                             "dsv3_routing_profile", "dsv3_profile"])
    ap.add_argument("--weights", choices=["dtype", "fp8", "w8a8", "mxfp4"], default="dtype",
                    help="expert weights in the activation dtype; E4M3 codes with per-row "
                         "scales (quantised once by the library before timing); those and "
                         "E4M3 activations inside the experts (W8A8); or MXFP4 codes with "
                         "per-32 block scales")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-streams", type=int, default=4,
                    help="host threads (each with its own stream, workspace and buffers) "
                         "taking alternate steps in the end-to-end timing")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the decode-shape leg of the default Mixtral-shaped run")
    ap.add_argument("--decode-calls", type=int, default=1000)
    return ap.parse_args(argv)


def workload_by_name(name):
    from sparse_mixture_experts_aux_b200 import inputs as I
    return {"mixtral": I.MIXTRAL, "deepseek_v3": I.DEEPSEEK_V3, "switch_zipf": I.SWITCH_ZIPF,
            "decode": I.MIXTRAL_DECODE, "tiny_fp32": I.TINY_F32,
            "mixtral_profile": I.MIXTRAL_PROFILE, "decode_profile": I.DECODE_PROFILE,
            "routing_profile": I.ROUTING_PROFILE,
            "dsv3_routing_profile": I.DSV3_ROUTING_PROFILE, "dsv3_profile": I.DSV3_PROFILE}[name]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def config_of(w, l2_note):
    return {"workload": w.name, "T": w.T, "d": w.d, "E": w.E, "d_e": w.d_e, "k": w.k,
            "d_s": w.d_s, "capacity_factor": w.capacity_factor, "router_bias": w.zipf_bias,
            "dtype_router": "f32", "l2": l2_note, "parallelism": "replicas"}


# --------------------------------------------------------------------------- ranks
def max_over_ranks(ms: float, device) -> float:
    """The slowest rank's time (all ranks call this at the same point)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, tokens_per_rank: int, steps: int, ms_max: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank * steps / (ms_max / 1e3)


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.out = None
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            sel = str(device_index)
        self.sel = sel

    def start(self):
        try:
            self.out = open(os.devnull, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.sel, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.12)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            return None
        rows = [r.split(",") for r in out.strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.strip() == "Active"})
        load = [s for s in sm if s > 0.5 * (max(mx) if mx else 1)] or sm
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# --------------------------------------------------------------------------- oracle timing
def oracle_sample_runner(w, x_batches_cpu, S):
    """Returns (step_fn, setup_seconds, threads): step_fn(i) runs the fp64 oracle
    on a sub-batch of S tokens of the workload and returns its wall time."""
    import numpy as np
    import torch
    from oracle import moe_oracle as O
    from sparse_mixture_experts_aux_b200.inputs import make_inputs, split_shared
    t0 = time.perf_counter()
    inp = make_inputs(w, device="cpu")
    W_r = inp["W_r"].numpy().astype(np.float64)
    experts = [tuple(t.float().numpy().astype(np.float64) for t in
                     (inp["W_g"][e], inp["W_u"][e], inp["W_d"][e])) for e in range(w.E)]
    shared = None
    if w.d_s:
        shared = tuple(t.float().numpy().astype(np.float64) for t in
                       split_shared(inp["W_shared"], w.d, w.d_s))
    bias = inp["router_bias"]
    del inp
    setup = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()

    def step(i):
        xb = x_batches_cpu[i % len(x_batches_cpu)]
        off = (i * S) % max(1, xb.shape[0] - S + 1)
        xs = xb[off:off + S]
        t = time.perf_counter()
        O.moe_forward(xs, W_r, lambda e: experts[e], w.k, w.capacity_factor, bias, shared)
        return time.perf_counter() - t

    return step, setup, threads


def run_reference(args, rank, world):
    """The oracle as it stands, on the host cores, on this arm's workload."""
    if rank != 0:
        return None
    import torch
    from sparse_mixture_experts_aux_b200.inputs import make_x
    w = workload_by_name(args.workload)
    S = 8 if w.T >= 8 else w.T
    xs = [make_x(w, "cpu", seed_offset=j) for j in range(2)]
    step, setup, threads = oracle_sample_runner(w, xs, S)
    for i in range(args.warmup):
        step(i)
    total = sum(step(args.warmup + i) for i in range(args.steps))
    value = S * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, "host memory (CPU oracle)"),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"{S} tokens of the workload per step (full routing and "
                                   f"experts for that sub-batch), weights pre-converted to "
                                   f"fp64 once ({setup:.1f} s, untimed)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    return line


# --------------------------------------------------------------------------- our arm
def step_work(w, counts, weights: str = "dtype"):
    """Algorithmic work of one step from its own routing counts: kept
    assignments, touched experts, FLOPs of the two GEMMs, and the bytes each
    GEMM and the whole layer must move at least (touched expert weights once,
    plus the rows a GEMM reads and writes; x in and y out for the layer).
    weights: "dtype", "fp8", "w8a8" (one byte per weight, 4 per weight row) or
    "mxfp4" (half a byte per weight, one per 32, 4 per weight row)."""
    fp8 = weights != "dtype"
    from sparse_mixture_experts_aux_b200 import _lib
    C = _lib.moe_capacity(w.T, w.E, w.k, w.capacity_factor)
    C = None if C < 0 else C
    kept_e = [int(c) if C is None else min(int(c), C) for c in counts]
    kept = sum(kept_e)
    touched = sum(1 for c in kept_e if c > 0)
    esz = 2 if w.dtype == "bf16" else 4
    # bytes per expert weight (+ 4 per weight row of scales when quantised)
    wsz = (0.5 + 1.0 / 32) if weights == "mxfp4" else (1 if fp8 else esz)
    sh = w.T if w.d_s else 0
    flops_up = 2 * kept * w.d * 2 * w.d_e + 2 * sh * w.d * 2 * w.d_s
    flops_down = 2 * kept * w.d_e * w.d + 2 * sh * w.d_s * w.d
    bytes_up = (touched * 2 * w.d * w.d_e * wsz + (touched * 2 * w.d_e * 4 if fp8 else 0)
                + 2 * w.d * w.d_s * esz + (kept * (w.d + w.d_e) + sh * (w.d + w.d_s)) * esz)
    bytes_down = (touched * w.d * w.d_e * wsz + (touched * w.d * 4 if fp8 else 0)
                  + w.d * w.d_s * esz + (kept * (w.d_e + w.d) + sh * (w.d_s + w.d)) * esz)
    w_bytes = (touched * 3 * w.d * w.d_e * wsz + (touched * 2 * (w.d_e + w.d) * 4 if fp8 else 0)
               + 3 * w.d * w.d_s * esz + w.E * w.d * 4)
    return dict(C=C, kept=kept, touched=touched, flops_up=flops_up, flops_down=flops_down,
                flops=flops_up + flops_down, bytes_up=bytes_up, bytes_down=bytes_down,
                w_bytes=w_bytes, act_bytes=2 * w.T * w.d * esz)


def launches_per_step(w, act_fp8: bool) -> int:
    """Kernels one forward call enqueues: the 7 steps, with the bf16 router step
    as two kernels (weight split + tensor-core logits) and, with E4M3
    activations, the x and H quantisers."""
    return 7 + (1 if w.dtype == "bf16" else 0) + (2 if act_fp8 else 0)


def kernel_roofline(flops, nbytes, ms, tensor_peak, hbm_peak):
    """The kernel's bound (the slower of its FLOPs at tensor peak and its
    algorithmic bytes at HBM bandwidth) and what it achieved against it."""
    if flops / (tensor_peak * 1e12) >= nbytes / (hbm_peak * 1e9):
        ach = flops / (ms / 1e3) / 1e12
        return dict(bound="tensor", achieved=ach, peak=tensor_peak, unit="TFLOP/s",
                    frac=ach / tensor_peak, algorithmic_per_launch=flops)
    ach = nbytes / (ms / 1e3) / 1e9
    return dict(bound="hbm", achieved=ach, peak=hbm_peak, unit="GB/s", frac=ach / hbm_peak,
                algorithmic_per_launch=nbytes)


def time_calls(call, n, stream, kev=None, local_rank=0):
    """Time n back-to-back calls on `stream` with CUDA events, sampling the
    clocks meanwhile; call(i, events) enqueues call i. Returns (ms, clocks)."""
    import torch
    clocks = ClockSampler(local_rank)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.2)
    t_start.record(stream)
    for i in range(n):
        call(i, kev[i].array if kev is not None else None)
    t_end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    return t_start.elapsed_time(t_end), clk


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from sparse_mixture_experts_aux_b200 import (KERNEL_NAMES, MOE_NUM_KERNELS, Workspace,
                                                 forward, _lib, moe_get_device_status,
                                                 quantize_fp8, quantize_mxfp4)
    from sparse_mixture_experts_aux_b200.events import KernelEvents
    from sparse_mixture_experts_aux_b200.inputs import MIXTRAL_DECODE, make_inputs, make_x
    from oracle import moe_oracle as O  # cpu_baseline leg only

    w = workload_by_name(args.workload)
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    inp = make_inputs(w.with_(seed=w.seed), device=str(dev))
    R = 8
    xs = [make_x(w, str(dev), seed_offset=100 * rank + j) for j in range(R)]
    ws = Workspace()
    y = torch.empty_like(xs[0])
    aux = torch.empty(1, dtype=torch.float32, device=dev)
    counts = torch.empty(w.E, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    fp8 = args.weights in ("fp8", "w8a8", "mxfp4")
    act_fp8 = args.weights == "w8a8"
    scales = bscales = None
    if args.weights == "mxfp4":  # one-off weight preparation, untimed
        parts, bparts = [], []
        for name in ("W_g", "W_u", "W_d"):
            inp[name], bs, rf = quantize_mxfp4(inp[name])
            parts.append(rf.reshape(-1))
            bparts.append(bs.reshape(-1))
        scales, bscales = torch.cat(parts), torch.cat(bparts)
        torch.cuda.synchronize()
    elif fp8:
        parts = []
        for name in ("W_g", "W_u", "W_d"):
            inp[name], sc = quantize_fp8(inp[name])
            parts.append(sc.reshape(-1))
        scales = torch.cat(parts)
        torch.cuda.synchronize()

    def call_on(xlist, yb, i, events=None):
        forward(xlist[i % len(xlist)], inp["W_r"], inp["W_g"], inp["W_u"], inp["W_d"],
                inp["W_shared"], k=w.k, capacity_factor=w.capacity_factor,
                router_bias=inp["router_bias"], d_s=w.d_s, workspace=ws, stream=stream,
                events=events, y=yb, aux=aux, counts=counts, weight_scales=scales,
                act_fp8=act_fp8, weight_block_scales=bscales)

    def barrier():
        if world > 1:
            dist.barrier()

    # per-step, per-kernel events recorded by the library on the launch stream
    kev = [KernelEvents(MOE_NUM_KERNELS) for _ in range(args.steps)]

    for i in range(max(3, args.warmup)):
        call_on(xs, y, i)
    torch.cuda.synchronize()
    if moe_get_device_status() != 0:
        raise RuntimeError("device-side wait timed out during warm-up")

    barrier()
    ms, clk = time_calls(lambda i, ev: call_on(xs, y, i, None), args.steps, stream, None,
                         local_rank)
    barrier()
    if moe_get_device_status() != 0:
        raise RuntimeError("device-side wait timed out in the timed region")
    # per-kernel breakdown: the same steps again, with the library's events around
    # each kernel (events between kernels stop them overlapping their launches,
    # so these steps are not part of the value's timing)
    time_calls(lambda i, ev: call_on(xs, y, i, ev), args.steps, stream, kev, local_rank)
    barrier()
    per_kernel = [statistics.mean(kev[i].elapsed_ms(j) for i in range(args.steps))
                  for j in range(MOE_NUM_KERNELS)]
    for kv in kev:
        kv.close()
    ms_max = max_over_ranks(ms, dev)

    wk = step_work(w, counts.cpu().numpy().astype("int64"), args.weights)
    peaks, peaks_src = load_peaks()
    # Headline tensor peak: the burst cuBLAS figure (a kernel timed in a short run at
    # full clock, as this one is); the sustained, power-capped figure is reported
    # beside it, labelled. E4M3 x E4M3: the bf16 figures times the nominal 4.5 / 2.25.
    ratio = 2.0 if act_fp8 else 1.0
    tensor_peak = peaks["bf16_tflops"] * ratio
    tensor_sust = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * ratio
    hbm_peak = peaks["hbm_gbs"]

    ms_step = ms_max / args.steps
    value = job_value(world, w.T, args.steps, ms_max)
    k_up, k_down = per_kernel[4], per_kernel[5]
    rl = kernel_roofline(wk["flops_up"], wk["bytes_up"], k_up, tensor_peak, hbm_peak)
    src = f"bf16_tflops{' x 2 (nominal e4m3/bf16 ratio)' if act_fp8 else ''} (of {peaks_src})"
    rl["peak_source"] = src if rl["bound"] == "tensor" else f"hbm_gbs (of {peaks_src})"
    if rl["bound"] == "tensor":
        rl["frac_of_sustained_peak"] = rl["achieved"] / tensor_sust
        rl["sustained_peak"] = tensor_sust
    mhz = (clk or {}).get("sm_mhz")
    rl["ms_per_launch"] = k_up
    rl["ms_x_sm_mhz"] = k_up * mhz if mhz else None  # clock-normalised duration
    # DRAM traffic of the dominant kernel: ncu's dram bytes over the algorithmic bytes on a
    # small case of the same kernel and per-expert load, times this launch's algorithmic
    # bytes; None where no capture of the kernel as built stands
    up_ratio = TRAFFIC_RATIO.get((args.workload, args.weights))
    rl["traffic"] = up_ratio[0] * wk["bytes_up"] if up_ratio is not None else None
    rl["traffic_source"] = ("ncu dram bytes / algorithmic bytes = %.3f on the %s, "
                            "times this launch's algorithmic bytes" % up_ratio
                            if up_ratio is not None else None)
    rl = {"kernel": KERNEL_NAMES[4], **rl}
    rl_down = kernel_roofline(wk["flops_down"], wk["bytes_down"], k_down, tensor_peak, hbm_peak)
    down_ratio = DOWN_TRAFFIC_RATIO.get((args.workload, args.weights))
    rl_down["traffic"] = down_ratio[0] * wk["bytes_down"] if down_ratio is not None else None
    roof_ms = max(wk["flops"] / (tensor_peak * 1e12),
                  (wk["w_bytes"] + wk["act_bytes"]) / (hbm_peak * 1e9)) * 1e3
    roof_ms_sust = max(wk["flops"] / (tensor_sust * 1e12),
                       (wk["w_bytes"] + wk["act_bytes"]) / (hbm_peak * 1e9)) * 1e3
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ("e4m3" if act_fp8 else ("bf16" if w.dtype == "bf16" else "f32")),
        "data": "synthetic",
        "config": dict(config_of(w, "inputs larger than L2: %.2f GB of expert weights streamed "
                                    "per step; x rotates over %d batches" % (wk["w_bytes"] / 1e9, R)),
                       weights=("e2m1 codes + e8m0 block scales (32) + fp32 row factors"
                                if args.weights == "mxfp4" else
                                "e4m3 codes + fp32 row scales" if fp8 else w.dtype),
                       activations="e4m3 rows + fp32 row scales in the experts" if act_fp8
                       else w.dtype),
        "roofline": rl,
        "down_roofline": {"kernel": KERNEL_NAMES[5], "ms_per_launch": k_down, **rl_down},
        "layer": {"active_tflops": wk["flops"] / (ms_step / 1e3) / 1e12,
                  "active_flops_per_step": wk["flops"], "touched_weight_bytes": wk["w_bytes"],
                  "roofline_ms": roof_ms, "frac_of_roofline": roof_ms / ms_step,
                  "frac_of_roofline_sustained_peak": roof_ms_sust / ms_step,
                  "hbm_gbs_weights": wk["w_bytes"] / (ms_step / 1e3) / 1e9,
                  "dropped_fraction": O.dropped_fraction(counts.cpu().numpy(), wk["C"], w.T, w.k),
                  "aux": float(aux.cpu()[0])},
        "kernel_ms": {KERNEL_NAMES[j]: per_kernel[j] for j in range(MOE_NUM_KERNELS)},
        "gpu_launches": launches_per_step(w, act_fp8) * args.steps * world,
        "clocks": clk,
        "when": datetime.datetime.now(datetime.timezone.utc).isoformat(timespec="seconds"),
    }

    # end to end through the host-buffer entry point: H2D x, forward, D2H y/aux/counts.
    # moe_forward_host_io returns once its stream is done, so several host threads (4 by
    # default), each with its own stream, workspace and buffers, take turns: one step's
    # copies overlap the others' kernels, and every step still copies its own x in and
    # its own y, aux and counts out inside the timed region.
    if not args.no_e2e:
        import threading
        ke = min(args.steps, 100)
        NSTR = args.e2e_streams
        streams = [stream] + [torch.cuda.Stream(dev) for _ in range(NSTR - 1)]
        x_host = [xs[j].cpu().pin_memory() for j in range(2)]
        nbytes = ws.buf.numel()
        fmt = (_lib.MOE_WEIGHTS_FP8_W8A8 if act_fp8 else
               _lib.MOE_WEIGHTS_MXFP4 if args.weights == "mxfp4" else
               _lib.MOE_WEIGHTS_FP8 if fp8 else _lib.MOE_WEIGHTS_DTYPE)
        bufs = []
        for sidx in range(NSTR):
            wsb = ws.buf if sidx == 0 else torch.empty(nbytes, dtype=torch.uint8, device=dev)
            b = dict(ws=wsb, x_dev=torch.empty_like(xs[0]), y_dev=torch.empty_like(xs[0]),
                     aux=torch.empty(1, dtype=torch.float32, device=dev),
                     counts=torch.empty(w.E, dtype=torch.int32, device=dev),
                     y_host=torch.empty_like(x_host[0]).pin_memory(),
                     aux_host=torch.empty(1, dtype=torch.float32).pin_memory(),
                     counts_host=torch.empty(w.E, dtype=torch.int32).pin_memory())
            b["dims"] = _lib.make_dims(w.T, w.d, w.d_e, w.d_s,
                                       _lib.MOE_BF16 if w.dtype == "bf16" else _lib.MOE_F32,
                                       inp["router_bias"], wsb, nbytes, streams[sidx].cuda_stream,
                                       weight_format=fmt, weight_scales=scales,
                                       weight_block_scales=bscales)
            bufs.append(b)

        def e2e_run(sidx, first, count):
            b = bufs[sidx]
            for i in range(first + sidx, first + count, NSTR):
                _lib.moe_forward_host_io(b["dims"], x_host[i % 2], b["x_dev"], inp["W_r"],
                                         inp["W_g"], inp["W_u"], inp["W_d"], inp["W_shared"],
                                         w.E, w.k, w.capacity_factor, b["y_dev"], b["y_host"],
                                         b["aux"], b["aux_host"], b["counts"], b["counts_host"])

        def e2e_steps(first, count):
            th = [threading.Thread(target=e2e_run, args=(sidx, first, count))
                  for sidx in range(NSTR)]
            for t in th:
                t.start()
            for t in th:
                t.join()

        e2e_steps(0, 4)
        torch.cuda.synchronize()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(streams[0])
        for sx in streams[1:]:
            sx.wait_event(e0)
        e2e_steps(0, ke)
        for sx in streams[1:]:
            done = torch.cuda.Event()
            done.record(sx)
            streams[0].wait_event(done)
        e1.record(streams[0])
        torch.cuda.synchronize()
        barrier()
        ems = max_over_ranks(e0.elapsed_time(e1), dev)
        esz = 2 if w.dtype == "bf16" else 4
        line["e2e"] = {"value": job_value(world, w.T, ke, ems), "unit": "tokens/s",
                       "h2d_bytes_per_step": w.T * w.d * esz,
                       "d2h_bytes_per_step": w.T * w.d * esz + 4 + 4 * w.E,
                       "steps": ke, "api": "moe_forward_host_io",
                       "streams": NSTR, "host_threads": NSTR}
        del bufs

    # the weight-streaming decode shape on the same weights: T = 32, one fresh x per call
    if args.workload == "mixtral" and not args.no_decode and args.decode_calls > 0:
        wd = MIXTRAL_DECODE.with_(dtype=w.dtype)
        n = args.decode_calls
        xd = make_x(wd, str(dev), seed_offset=5000 + 100 * rank, T=wd.T * n).view(n, wd.T, wd.d)
        yd = torch.empty(wd.T, wd.d, dtype=xd.dtype, device=dev)
        xl = [xd[i] for i in range(n)]
        cd = torch.empty(wd.E, dtype=torch.int32, device=dev)

        def dcall(i, events=None):
            forward(xl[i], inp["W_r"], inp["W_g"], inp["W_u"], inp["W_d"], None, k=wd.k,
                    workspace=ws, stream=stream, events=events, y=yd, aux=aux, counts=cd,
                    weight_scales=scales, act_fp8=act_fp8, weight_block_scales=bscales)

        for i in range(max(3, args.warmup)):
            dcall(i)
        torch.cuda.synchronize()
        dkev = [KernelEvents(MOE_NUM_KERNELS) for _ in range(n)]
        barrier()
        dms, dclk = time_calls(lambda i, ev: dcall(i, None), n, stream, None, local_rank)
        barrier()
        if moe_get_device_status() != 0:
            raise RuntimeError("device-side wait timed out in the decode leg")
        time_calls(dcall, n, stream, dkev, local_rank)  # per-kernel breakdown, as above
        barrier()
        dk = [statistics.mean(dkev[i].elapsed_ms(j) for i in range(n))
              for j in range(MOE_NUM_KERNELS)]
        for kv in dkev:
            kv.close()
        dms_max = max_over_ranks(dms, dev)
        dwk = step_work(wd, cd.cpu().numpy().astype("int64"), args.weights)
        d_ms = dms_max / n
        d_roof = max(dwk["flops"] / (tensor_peak * 1e12),
                     (dwk["w_bytes"] + dwk["act_bytes"]) / (hbm_peak * 1e9)) * 1e3
        line["decode"] = {
            "workload": wd.name, "calls": n, "distinct_x": n, "ms_per_call": d_ms,
            "tokens_per_s": job_value(world, wd.T, n, dms_max),
            "touched_weight_bytes": dwk["w_bytes"],
            "hbm_gbs": (dwk["w_bytes"] + dwk["act_bytes"]) / (d_ms / 1e3) / 1e9,
            "hbm_peak_gbs": hbm_peak, "roofline_ms": d_roof, "frac_of_roofline": d_roof / d_ms,
            "gate_up": {"ms_per_launch": dk[4],
                        **kernel_roofline(dwk["flops_up"], dwk["bytes_up"], dk[4], tensor_peak,
                                          hbm_peak)},
            "down": {"ms_per_launch": dk[5],
                     **kernel_roofline(dwk["flops_down"], dwk["bytes_down"], dk[5], tensor_peak,
                                       hbm_peak)},
            "kernel_ms": {KERNEL_NAMES[j]: dk[j] for j in range(MOE_NUM_KERNELS)},
            "gpu_launches": launches_per_step(wd, act_fp8) * n * world,
            "clocks": dclk,
            "l2": "weights (%.2f GB) larger than L2; each call reads its own x" % (dwk["w_bytes"] / 1e9),
        }
        del xd, xl

    # the oracle on the host cores, bounded sample, rank 0 at N=1 only
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        xs_cpu = [xs[0].cpu()]
        del inp
        torch.cuda.empty_cache()
        S = 8 if w.T >= 8 else w.T
        step, setup, threads = oracle_sample_runner(w, xs_cpu, S)
        times = []
        budget = 20.0
        while sum(times) < budget and len(times) < 200:
            times.append(step(len(times)))
        line["cpu_baseline"] = {
            "value": S * len(times) / sum(times), "unit": "tokens/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{len(times)} sub-batches of {S} tokens of the workload (full routing and "
                      f"experts per sub-batch), fp64, weights pre-converted once (untimed)"}
    return line


# --------------------------------------------------------------------------- launch
def _free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_entry(rank, world, port, backend, fn, timeout_s):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    import torch
    import torch.distributed as dist
    kw = {}
    if backend == "nccl":
        torch.cuda.set_device(rank)
        kw["device_id"] = torch.device("cuda", rank)
    dist.init_process_group(backend, rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=timeout_s), **kw)
    try:
        fn(rank, world)
    finally:
        dist.destroy_process_group()


def launch_local_ranks(n: int, fn, backend: str = "nccl", timeout_s: int = 300) -> list:
    """Run fn(rank, world) in n spawned processes on this node, one per GPU
    (LOCAL_RANK = rank), with a process group over `backend` and a rendezvous on
    127.0.0.1. Returns the processes' exit codes."""
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_entry, args=(r, n, port, backend, fn, timeout_s))
             for r in range(n)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout_s + 600)
        if p.is_alive():
            p.kill()
            p.join()
    return [p.exitcode for p in procs]


def run_rank(args, rank, world):
    """One rank of our arm: run the benchmark, rank 0 prints the line."""
    line = run_ours(args, rank, world, int(os.environ.get("LOCAL_RANK", rank)))
    if rank == 0:
        print(json.dumps(line), flush=True)


def main(argv=None):
    args = parse_args(argv)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        import functools
        codes = launch_local_ranks(args.gpus, functools.partial(run_rank, args), "nccl")
        return 0 if all(c == 0 for c in codes) else 1
    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
