#!/usr/bin/env python
"""Benchmark of the routed MoE FFN forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload mixtral]
    python bench.py --impl reference ...   # the fp64 CPU oracle, timed on host cores

One step = one moe_forward call over one batch of T tokens: router logits,
routing, scan, scatter, gate/up GEMM + SwiGLU, down GEMM + gate scaling,
combine. Weights and a ring of fresh x batches are resident in HBM before the
timed region; the expert weights (2.8 GB for the Mixtral-shaped layer) are
larger than L2, so no L2 flush is needed between steps. Under torchrun every
rank runs its own replica on its own GPU ("replicas only": the layer has no
exchange step); the job value is the tokens of all ranks over the slowest
rank's device time. Rank 0 prints one JSON line.
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


# (workload, weights) -> DRAM bytes / algorithmic bytes of the gate/up kernel, from one ncu
# capture of that kernel as built (profiles/); absent = not captured for the current build.
TRAFFIC_RATIO = {("mixtral", "dtype"): 539.386880 / 545.259520}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mixtral",
                    choices=["mixtral", "deepseek_v3", "switch_zipf", "decode", "tiny_fp32",
                             "mixtral_profile", "decode_profile"])
    ap.add_argument("--weights", choices=["dtype", "fp8", "w8a8"], default="dtype",
                    help="expert weights in the activation dtype; E4M3 codes with per-row "
                         "scales (quantised once by the library before timing); or those and "
                         "E4M3 activations inside the experts (W8A8)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


def workload_by_name(name):
    from sparse_mixture_experts_aux_b200 import inputs as I
    return {"mixtral": I.MIXTRAL, "deepseek_v3": I.DEEPSEEK_V3, "switch_zipf": I.SWITCH_ZIPF,
            "decode": I.MIXTRAL_DECODE, "tiny_fp32": I.TINY_F32,
            "mixtral_profile": I.MIXTRAL_PROFILE, "decode_profile": I.DECODE_PROFILE}[name]


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
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from sparse_mixture_experts_aux_b200 import (KERNEL_NAMES, MOE_NUM_KERNELS, Workspace,
                                                 forward, _lib, moe_get_device_status,
                                                 quantize_fp8)
    from sparse_mixture_experts_aux_b200.events import KernelEvents
    from sparse_mixture_experts_aux_b200.inputs import make_inputs, make_x
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
    fp8 = args.weights in ("fp8", "w8a8")
    act_fp8 = args.weights == "w8a8"
    scales = None
    if fp8:  # one-off weight preparation, untimed
        parts = []
        for name in ("W_g", "W_u", "W_d"):
            inp[name], sc = quantize_fp8(inp[name])
            parts.append(sc.reshape(-1))
        scales = torch.cat(parts)
        torch.cuda.synchronize()

    def call(i, events=None):
        forward(xs[i % R], inp["W_r"], inp["W_g"], inp["W_u"], inp["W_d"], inp["W_shared"],
                k=w.k, capacity_factor=w.capacity_factor, router_bias=inp["router_bias"],
                d_s=w.d_s, workspace=ws, stream=stream, events=events, y=y, aux=aux,
                counts=counts, weight_scales=scales, act_fp8=act_fp8)

    def barrier():
        if world > 1:
            dist.barrier()

    # per-step, per-kernel events recorded by the library on the launch stream
    kev = [KernelEvents(MOE_NUM_KERNELS) for _ in range(args.steps)]

    for i in range(max(3, args.warmup)):
        call(i)
    torch.cuda.synchronize()
    if moe_get_device_status() != 0:
        raise RuntimeError("device-side wait timed out during warm-up")

    clocks = ClockSampler(local_rank)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.2)
    t_start.record(stream)
    for i in range(args.steps):
        call(i, kev[i].array)
    t_end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier()
    ms = t_start.elapsed_time(t_end)
    if moe_get_device_status() != 0:
        raise RuntimeError("device-side wait timed out in the timed region")
    per_kernel = [statistics.mean(kev[i].elapsed_ms(j) for i in range(args.steps))
                  for j in range(MOE_NUM_KERNELS)]
    for kv in kev:
        kv.close()
    ms_max = max_over_ranks(ms, dev)

    # algorithmic work of one step, from this step's own routing counts
    cnt = counts.cpu().numpy().astype("int64")
    C = _lib.moe_capacity(w.T, w.E, w.k, w.capacity_factor)
    C = None if C < 0 else C
    kept = int(cnt.sum() if C is None else sum(min(int(c), C) for c in cnt))
    touched = int(sum(1 for c in cnt if (c if C is None else min(int(c), C)) > 0))
    esz = 2 if w.dtype == "bf16" else 4
    wsz = 1 if fp8 else esz  # bytes per expert weight (+ 4 per row of scales with FP8)
    flops_up = 2 * kept * w.d * 2 * w.d_e + (2 * w.T * w.d * 2 * w.d_s if w.d_s else 0)
    flops_down = 2 * kept * w.d_e * w.d + (2 * w.T * w.d_s * w.d if w.d_s else 0)
    flops_active = flops_up + flops_down
    w_bytes = (touched * 3 * w.d * w.d_e * wsz + (touched * 2 * (w.d_e + w.d) * 4 if fp8 else 0)
               + 3 * w.d * w.d_s * esz + w.E * w.d * 4)
    act_bytes = 2 * w.T * w.d * esz
    peaks, peaks_src = load_peaks()
    tensor_peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    if act_fp8:  # E4M3 x E4M3: the bf16 figure times the nominal 4.5 / 2.25 ratio
        tensor_peak *= 2.0
    hbm_peak = peaks["hbm_gbs"]

    ms_step = ms_max / args.steps
    value = job_value(world, w.T, args.steps, ms_max)
    k_up = per_kernel[4]
    # the gate/up kernel's own roofline: its FLOPs at tensor peak vs its
    # algorithmic bytes (touched gate+up weights, permuted rows in, H out) at HBM
    bytes_up = (touched * 2 * w.d * w.d_e * wsz + (touched * 2 * w.d_e * 4 if fp8 else 0)
                + (2 * w.d * w.d_s * esz if w.d_s else 0)
                + (kept + (w.T if w.d_s else 0)) * (w.d + w.d_e) * esz)
    up_bound = "tensor" if flops_up / (tensor_peak * 1e12) >= bytes_up / (hbm_peak * 1e9) else "hbm"
    if up_bound == "tensor":
        achieved, peak, unit, work = flops_up / (k_up / 1e3) / 1e12, tensor_peak, "TFLOP/s", flops_up
        peak_note = (f"bf16_tflops_sustained x 2 (nominal e4m3/bf16 ratio; of {peaks_src})"
                     if act_fp8 else f"bf16_tflops_sustained (of {peaks_src})")
    else:
        achieved, peak, unit, work = bytes_up / (k_up / 1e3) / 1e9, hbm_peak, "GB/s", bytes_up
        peak_note = f"hbm_gbs (of {peaks_src})"
    # DRAM traffic of the dominant kernel: ncu's dram bytes over the algorithmic bytes on a
    # small case of the same kernel and per-expert load, times this launch's algorithmic
    # bytes (profiles/tc_grouped_gemm_mixtral_shape.md); None where no capture of the
    # kernel as built stands
    traffic_ratio = TRAFFIC_RATIO.get((args.workload, args.weights))
    traffic = traffic_ratio * bytes_up if traffic_ratio is not None else None
    roofline_ms = max(flops_active / (tensor_peak * 1e12), (w_bytes + act_bytes) / (hbm_peak * 1e9)) * 1e3
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ("e4m3" if act_fp8 else ("bf16" if w.dtype == "bf16" else "f32")),
        "data": "synthetic",
        "config": dict(config_of(w, "inputs larger than L2: %.2f GB of expert weights streamed "
                                    "per step; x rotates over %d batches" % (w_bytes / 1e9, R)),
                       weights="e4m3 codes + fp32 row scales" if fp8 else w.dtype,
                       activations="e4m3 rows + fp32 row scales in the experts" if act_fp8
                       else w.dtype),
        "roofline": {"bound": up_bound, "kernel": KERNEL_NAMES[4], "achieved": achieved,
                     "peak": peak, "unit": unit, "frac": achieved / peak, "traffic": traffic,
                     "traffic_source": ("ncu dram bytes / algorithmic bytes = %.3f on the "
                                        "T=1024 E=2 case, times this launch's algorithmic "
                                        "bytes" % traffic_ratio) if traffic is not None else None,
                     "algorithmic_per_launch": work, "peak_source": peak_note},
        "layer": {"active_tflops": flops_active / (ms_step / 1e3) / 1e12,
                  "active_flops_per_step": flops_active, "touched_weight_bytes": w_bytes,
                  "roofline_ms": roofline_ms, "frac_of_roofline": roofline_ms / ms_step,
                  "hbm_gbs_weights": w_bytes / (ms_step / 1e3) / 1e9,
                  "dropped_fraction": O.dropped_fraction(cnt, C, w.T, w.k),
                  "aux": float(aux.cpu()[0])},
        "kernel_ms": {KERNEL_NAMES[j]: per_kernel[j] for j in range(MOE_NUM_KERNELS)},
        # W8A8 adds the x and H quantisers to the 7 kernels of a step
        "gpu_launches": (MOE_NUM_KERNELS + (2 if act_fp8 else 0)) * args.steps * world,
        "clocks": clk,
        "when": datetime.datetime.now(datetime.timezone.utc).isoformat(timespec="seconds"),
    }

    # end to end through the host-buffer entry point: H2D x, forward, D2H y/aux/counts.
    # moe_forward_host_io returns once its stream is done, so two host threads, each
    # with its own stream, workspace and buffers, take alternate steps: one step's copies
    # overlap the other's kernels, and every step still copies its own x in and its own
    # y, aux and counts out inside the timed region.
    if not args.no_e2e:
        import threading
        ke = min(args.steps, 100)
        NSTR = 2
        streams = [stream, torch.cuda.Stream(dev)]
        x_host = [xs[j].cpu().pin_memory() for j in range(2)]
        nbytes = ws.buf.numel()
        fmt = (_lib.MOE_WEIGHTS_FP8_W8A8 if act_fp8 else
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
                                       weight_format=fmt, weight_scales=scales)
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
        streams[1].wait_event(e0)
        e2e_steps(0, ke)
        done1 = torch.cuda.Event()
        done1.record(streams[1])
        streams[0].wait_event(done1)
        e1.record(streams[0])
        torch.cuda.synchronize()
        barrier()
        ems = max_over_ranks(e0.elapsed_time(e1), dev)
        line["e2e"] = {"value": job_value(world, w.T, ke, ems), "unit": "tokens/s",
                       "h2d_bytes_per_step": w.T * w.d * esz,
                       "d2h_bytes_per_step": w.T * w.d * esz + 4 + 4 * w.E,
                       "steps": ke, "api": "moe_forward_host_io",
                       "streams": NSTR, "host_threads": NSTR}

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


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0
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
