#!/usr/bin/env python
"""Benchmark of the Grok-1 MoE feed-forward layer on B200: tokens/s at the Grok-1
shape (d_model 6144, ffn 32768, 8 experts, top-2, int8 weights) and the fraction
of the HBM / bf16 tensor roofline reached by the dominant kernel.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill|decode|skewed|stacked]
    python bench.py --impl reference ...      # the fp64 CPU oracle on the host cores

One step = one pass of the whole layer (router, dispatch, gather, up-projection,
down-projection, combine) over one batch of T synthetic tokens; the stacked
workload's step is its four residual blocks.  The headline line is the prefill
workload (T = 8192, one full context: the largest configuration, bound by the bf16
tensor pipe); with no --workload it also carries a `workloads` object with the
decode (HBM-bound), skewed-routing and stacked-block workloads and the API weight
layout's decode and prefill, each measured the same way.

Timing: W untimed warm-up steps, then R repeats of a region of exactly K steps,
each bracketed by a barrier and a device synchronisation and timed with CUDA events
on the launching stream; the reported time is the median region.  After each timed
region the same K steps run again with events around every launch: the per-kernel
durations (the median over those regions) behind the roofline come from the same clock
and power-cap conditions as the timed regions, which carry no events.  Inputs are
resident in HBM when a region starts; the layer weights (4.8 GB per layer) are
larger than L2, so every step streams them from HBM.  Under torchrun each rank runs
an independent replica on its own GPU and its own token batch (no collective on the
data path); the reported value is all ranks' tokens over the slowest rank's time.
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
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/sec at Grok-1 shape; % of HBM / bf16 tensor-pipe roofline"
KERNELS = ("router", "dispatch", "gather", "up_proj", "down_proj", "combine", "prenorm", "route_small")
DATA = "synthetic (seeded; random-init int8 weights of the Grok-1 MoE shape)"

# sub-records of the default run: (record name, workload, weight layout)
SUBRECORDS = (("decode", "decode", "packed"), ("skewed", "skewed", "packed"), ("stacked", "stacked", "packed"),
              ("decode_api_layout", "decode", "in_out"), ("prefill_api_layout", "prefill", "in_out"))
TIMED_SECONDS = 1.5       # repeats of the K-step region fill about this much device time
SUB_CPU_SECONDS = 5.0     # oracle budget of each sub-record's CPU baseline


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=None)
    p.add_argument("--warmup", type=int, default=None)
    p.add_argument("--impl", choices=("native", "reference"), default="native")
    p.add_argument("--workload", default=None, choices=("decode", "prefill", "skewed", "stacked", "tiny"),
                   help="one workload only (default: prefill as the headline plus the sub-records)")
    p.add_argument("--repeats", type=int, default=None, help="timed K-step regions (default: ~1.5 s of them)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the headline's oracle sample")
    # smaller variants of a workload for profiler captures (never a bench line)
    p.add_argument("--tokens", type=int, default=None, help="override T")
    p.add_argument("--ffn", type=int, default=None, help="override the FFN width")
    p.add_argument("--skip-extras", action="store_true", help="skip the per-kernel and end-to-end passes")
    p.add_argument("--scale-block", type=int, choices=(0, 128), default=0,
                   help="weight scale format: 0 per output channel, 128 per block of 128 inputs (packed layout)")
    p.add_argument("--layout", choices=("packed", "in_out"), default="packed",
                   help="weight layout: packed = tiles written once at load (TMEM path); in_out = as drawn")
    p.add_argument("--cta-pairs", type=int, choices=(0, 1, 2, 3), default=None,
                   help="GEMMs on CTA pairs: 0 never, 1 the down-projection of 128-route plans (library default), "
                        "2 both GEMMs of those plans, 3 also small batches")
    p.add_argument("--no-cta-pairs", dest="cta_pairs", action="store_const", const=0,
                   help="the same as --cta-pairs 0")
    p.add_argument("--parallel", choices=("replicas", "ep"), default="replicas",
                   help="several GPUs: independent replicas (default), or experts spread over the ranks "
                        "(each rank E/N experts and its own tokens; all-to-all exchanges over NCCL)")
    return p.parse_args(argv)


def default_steps(workload):
    return {"decode": (200, 10), "stacked": (50, 5), "prefill": (20, 5), "skewed": (20, 5),
            "tiny": (200, 10)}[workload]


def repeats_for(ms_per_step: float, steps: int, requested=None) -> int:
    """Timed regions of `steps` steps: enough to fill about TIMED_SECONDS (so that the clock
    sampler sees the timed regions themselves), at least 3, at most 200."""
    if requested:
        return max(1, int(requested))
    region_s = max(ms_per_step, 1e-3) * steps / 1e3
    return int(min(200, max(3, math.ceil(TIMED_SECONDS / region_s))))


# ---- distributed plumbing --------------------------------------------------------

def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 or "MASTER_ADDR" in os.environ:   # under torchrun (a one-rank group included)
        import datetime
        import torch.distributed as dist
        backend = os.environ.get("MOE_BENCH_BACKEND", "nccl")
        if backend == "nccl":
            import torch
            torch.cuda.set_device(local)
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world <= 1:
        return value
    import torch
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


def job_value(tokens_per_rank: int, world: int, ms_per_rank: float, device=None):
    """Whole-job throughput of `world` replicas: all ranks' tokens over the slowest rank's
    time per step.  Returns (tokens/s, slowest ms per step); every rank gets the same pair."""
    ms_max = max_over_ranks(ms_per_rank, world, device)
    return tokens_per_rank * world / (ms_max / 1e3), ms_max


def dist_teardown(world: int):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()


# ---- clocks sampled during the timed region --------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
            return
        self.th = threading.Thread(target=self._read, daemon=True)
        self.th.start()
        t_end = time.time() + 5.0
        while not self.lines and time.time() < t_end and self.proc.poll() is None:
            time.sleep(0.02)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.th.join(timeout=2)
        return summarize_clocks(self.lines, self.t0, self.t1)


def summarize_clocks(lines, t0, t1):
    """nvidia-smi rows (time, csv line) -> median SM clock, max clock and the throttle reasons
    seen, over the rows inside [t0, t1] (all rows when none falls inside)."""
    rows = []
    for ts, line in lines:
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            rows.append((ts, float(parts[1]), float(parts[2]), parts[4:]))
        except ValueError:
            continue
    if not rows:
        return None
    inside = [r for r in rows if t0 and t1 and t0 <= r[0] <= t1]
    use = inside if inside else rows
    names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    reasons = set()
    for r in use:
        for nm, v in zip(names, r[3][1:]):
            if v.lower() == "active":
                reasons.add(nm)
    return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
            "reasons": sorted(reasons), "samples": len(use),
            "window": "timed region" if inside else "whole run (timed region shorter than one sample)"}


# ---- roofline bookkeeping ----------------------------------------------------------

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


GEMM_SOURCES = {"packed": ("gemm_ts.cu", "gemm_ts2.cu", "gemm_common.cuh", "ptx.cuh", "kernels.cuh"),
                "in_out": ("gemm.cu", "gemm_common.cuh", "ptx.cuh", "kernels.cuh")}


def kernel_source_hash(layout):
    """Hash of the GEMM sources of a weight layout: a recorded DRAM-traffic figure holds only for them."""
    h = hashlib.sha256()
    for name in GEMM_SOURCES[layout]:
        with open(os.path.join(ROOT, "mixture_experts_softmax_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload, layout, kernel, variant):
    """DRAM bytes per full-size launch from the committed ncu summary (profiles/traffic.json),
    or None: no record for this workload, a variant of it (resized, other scale format), or
    GEMM sources changed since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if variant or not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    ent = rec.get(f"{workload}/{layout}/{kernel}")
    if not ent or ent.get("source_hash") != kernel_source_hash(layout):
        return None
    return ent.get("bytes_per_launch")


def algorithmic_work(w, T, n_touched, counts, kblock=0):
    """Per-launch algorithmic bytes and FLOPs of the up- and down-projection kernels
    (kblock: 0 = one bf16 scale per output channel, else one per block of kblock inputs)."""
    d, F = w.d, w.F
    R = 2 * T
    up_scales = 2 * 2 * F * (d // kblock if kblock else 1)
    dn_scales = 2 * d * (F // kblock if kblock else 1)
    up_bytes = n_touched * (2 * d * F + up_scales) + R * d * 2 + R * F * 2
    dn_bytes = n_touched * (F * d + dn_scales) + R * F * 2 + R * d * 4
    up_flops = 2.0 * R * d * F * 2
    dn_flops = 2.0 * R * F * d
    return dict(up_bytes=up_bytes, dn_bytes=dn_bytes, up_flops=up_flops, dn_flops=dn_flops)


def roofline_of(workload, layout, work, up_ms, peaks, peak_src, variant):
    """The dominant kernel (the up-projection) against its bound: the sustained bf16 GEMM figure
    for the tensor-bound workloads (its time comes from back-to-back steps under the power cap;
    the burst fraction is context), measured copy bandwidth for the HBM-bound ones."""
    if workload in ("prefill", "skewed"):
        achieved = work["up_flops"] / (up_ms / 1e3) / 1e12
        peak = peaks["bf16_tflops_sustained"]
        return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "frac_of_burst": achieved / peaks["bf16_tflops"], "kernel": "up_proj",
                "peak_source": f"{peak_src} bf16_tflops_sustained (kernel timed inside a long step loop)",
                "traffic": recorded_traffic(workload, layout, "up_proj", variant),
                "algorithmic_flops_per_launch": work["up_flops"], "launch_ms": up_ms}
    achieved = work["up_bytes"] / (up_ms / 1e3) / 1e9
    peak = peaks["hbm_gbs"]
    return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "kernel": "up_proj", "peak_source": f"{peak_src} hbm_gbs (copy)",
            "traffic": recorded_traffic(workload, layout, "up_proj", variant),
            "algorithmic_bytes_per_launch": work["up_bytes"], "launch_ms": up_ms}


# ---- the CUDA path -------------------------------------------------------------------

def bench_workload(name, args, world, rank, dev, layout, cpu_seconds, with_cpu):
    """One workload, measured: the K-step regions, the per-kernel pass, the end-to-end pass
    with host buffers and (rank 0, one process) the oracle on the host cores.  Returns the
    record and the number of this library's kernel launches per step."""
    import torch
    import moe_synth
    import mixture_experts_softmax_b200 as moe

    w = moe_synth.WORKLOADS[name]
    if args.tokens or args.ffn:
        import dataclasses
        w = dataclasses.replace(w, T=args.tokens or w.T, F=args.ffn or w.F, name=w.name + "_resized")
    variant = bool(args.tokens or args.ffn or args.scale_block)
    ks, ws = default_steps(name)
    K = args.steps if args.steps is not None else ks
    W = max(3, args.warmup if args.warmup is not None else ws)
    inp = moe_synth.make_inputs(w, device=dev, seed=w.seed)
    if world > 1:   # each replica gets its own token batch; the layer weights are the same model
        g = moe_synth.generator(w.seed + 1000 + rank, dev)
        inp.x = moe_synth.draw_tokens(w.T, w.d, g, dev)
    T = w.T
    layers = inp.layers
    if args.scale_block:   # per-block scale format: the same weights, one scale row per 128 inputs
        gs = moe_synth.generator(w.seed + 2000, dev)
        layers = [moe_synth.block_scales(l, args.scale_block, gs) for l in layers]
    # the oracle reads the layer as drawn ([E, in, out]); keep host copies before any repacking
    cpu_layers = [{k: v.cpu() for k, v in l.items()} for l in layers] if with_cpu else None
    stream = torch.cuda.current_stream(dev)

    h = moe.MoELayer(w.d, w.F, w.E, w.k)
    if args.cta_pairs is not None:
        moe.check(moe.moe_set_cta_pairs(h.h, args.cta_pairs))
    moe.check(moe.moe_set_router_bias(h.h, inp.bias))
    moe.check(moe.moe_set_scale_block(h.h, args.scale_block))
    if layout == "packed":
        # one-time weight-load step, outside every timed region: K-major int8 copies
        moe.check(moe.moe_set_weight_layout(h.h, moe.MOE_LAYOUT_PACKED))
        drawn = layers
        layers = [moe.pack_layer(h.h, l) for l in drawn]
        torch.cuda.synchronize(dev)
        for l in drawn:
            for k in ("wl", "wv", "w1"):
                l[k] = None
        del drawn
        inp.layers = None
        torch.cuda.empty_cache()
    out = torch.empty_like(inp.x)
    res0 = inp.x.clone()
    hio = torch.empty_like(inp.x)

    def step():
        if w.blocks:
            hio.copy_(res0)
            for b in range(w.blocks):
                moe.check(moe.moe_block_forward(h.h, T, hio, inp.gammas[b]["pre"], inp.gammas[b]["post"], w.eps,
                                                *moe.layer_args(layers[b]), stream))
        else:
            moe.check(moe.moe_forward(h.h, T, inp.x, *moe.layer_args(layers[0]), out, stream))

    # warm-up (timed only to size the repeats)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(W):
        step()
    e1.record(stream)
    moe.check(moe.moe_sync_status(h.h, stream))
    R = repeats_for(e0.elapsed_time(e1) / W, K, args.repeats)
    R = int(max_over_ranks(R, world, dev))   # every rank runs the same number of regions

    # R regions of exactly K steps, device-timed; the median region is reported.  Unless the extras
    # are skipped, each timed region is followed by the same K steps with events around every launch
    # (moe_set_profiling), so that the per-kernel durations behind the roofline come from the same
    # clock and power-cap conditions as the timed regions; the timed regions themselves carry no
    # events.
    clocks = ClockSampler(dev.index) if rank == 0 else None
    if clocks:
        clocks.start()
    region_ms = []
    kernel_regions = []   # per profiled region: {kernel: (total ms, launches)}
    for r in range(R):
        barrier(world, dev)
        torch.cuda.synchronize(dev)
        if clocks and r == 0:
            clocks.mark("t0")
        e0.record(stream)
        for _ in range(K):
            step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        region_ms.append(e0.elapsed_time(e1))
        if not args.skip_extras:
            moe.check(moe.moe_set_profiling(h.h, True))
            moe.moe_get_kernel_times(h.h)
            for _ in range(K):
                step()
            torch.cuda.synchronize(dev)
            rc, kt = moe.moe_get_kernel_times(h.h)
            moe.check(rc)
            moe.check(moe.moe_set_profiling(h.h, False))
            kernel_regions.append(kt)
    if clocks:
        clocks.mark("t1")
    barrier(world, dev)
    clk = clocks.stop() if clocks else None
    moe.check(moe.moe_sync_status(h.h, stream), "device status after the timed region")
    ms = statistics.median(region_ms) / K
    value, ms_max = job_value(T, world, ms, dev)
    tokens = T * world
    rec = {"value": value, "unit": "tokens/s", "ms_per_step": ms_max, "steps": K, "warmup": W, "repeats": R,
           "region_ms": {"min": min(region_ms), "median": statistics.median(region_ms), "max": max(region_ms)},
           "config": {"workload": w.name, "T_per_gpu": T, "d_model": w.d, "ffn": w.F, "experts": w.E,
                      "top_k": w.k, "blocks": w.blocks or 1,
                      "router_bias": w.bias,
                      "weights": "int8 + bf16 " + ("scales per block of %d inputs" % args.scale_block
                                                   if args.scale_block else "per-output-channel scales") +
                                 ", layout " + layout +
                                 (" (packed once at load, untimed)" if layout == "packed" else " (as drawn)"),
                      "parallelism": f"replicas x{world}", "tile_routes": moe.moe_plan(h.h, T)[1],
                      "cta_pairs": "library default" if args.cta_pairs is None else args.cta_pairs,
                      "down_splits": moe.moe_plan(h.h, T)[2]},
           "clocks": clk}

    if args.skip_extras:
        h.close()
        rec["note"] = "profiling variant: no per-kernel or end-to-end pass"
        return rec, None

    per_launch, launches_per_step = kernel_times_over_regions(kernel_regions, K)

    # routing of the last step -> experts that received tokens
    offsets = torch.empty(w.E + 1, dtype=torch.int32, device=dev)
    moe.check(moe.moe_get_routing(h.h, None, None, offsets, None, stream))
    off = offsets.cpu().tolist()
    counts = [off[e + 1] - off[e] for e in range(w.E)]
    n_touched = sum(1 for c in counts if c > 0)

    # end to end through the public API with host buffers: pinned input in, result out, every step
    x_host = inp.x.cpu().pin_memory()
    out_host = torch.empty_like(x_host).pin_memory()
    if w.blocks:
        def e2e_step():   # the residual stream in, four blocks, the residual stream out
            hio.copy_(x_host, non_blocking=True)
            for b in range(w.blocks):
                moe.check(moe.moe_block_forward(h.h, T, hio, inp.gammas[b]["pre"], inp.gammas[b]["post"], w.eps,
                                                *moe.layer_args(layers[b]), stream))
            out_host.copy_(hio, non_blocking=True)
        api = "moe_block_forward x%d with pinned host copies of the residual stream" % w.blocks
    else:
        # successive calls overlap each input copy with the previous call's layer
        moe.check(moe.moe_set_host_overlap(h.h, 1))

        def e2e_step():
            moe.check(moe.moe_forward_host(h.h, T, x_host, *moe.layer_args(layers[0]), out_host, stream))
        api = "moe_forward_host (moe_set_host_overlap on)"
    # the region ends once the last result has reached host memory (the output copies of
    # host-overlap forwards run on a stream of the handle)
    e2e_end = (lambda: None) if w.blocks else (lambda: moe.check(moe.moe_host_wait(h.h, stream)))
    for _ in range(max(1, W // 2)):
        e2e_step()
    # timed like the device figure: R regions of K steps, the median region, so that both run for
    # about as long under the same power cap
    e2e_clocks = ClockSampler(dev.index) if rank == 0 else None
    if e2e_clocks:
        e2e_clocks.start()
    e2e_regions = []
    for r in range(R):
        barrier(world, dev)
        torch.cuda.synchronize(dev)
        if e2e_clocks and r == 0:
            e2e_clocks.mark("t0")
        e0.record(stream)
        for _ in range(K):
            e2e_step()
        e2e_end()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_regions.append(e0.elapsed_time(e1))
    if e2e_clocks:
        e2e_clocks.mark("t1")
    barrier(world, dev)
    e2e_clk = e2e_clocks.stop() if e2e_clocks else None
    e2e_ms = max_over_ranks(statistics.median(e2e_regions) / K, world, dev)
    moe.check(moe.moe_sync_status(h.h, stream))
    nb = T * w.d * 2
    rec["e2e"] = {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": nb,
                  "d2h_bytes_per_step": nb, "ms_per_step": e2e_ms, "repeats": R, "api": api, "clocks": e2e_clk}

    peaks, peak_src = measured_peaks()
    work = algorithmic_work(w, T, n_touched, counts, args.scale_block)
    rec["roofline"] = roofline_of(name, layout, work, per_launch["up_proj"], peaks, peak_src, variant)
    layer_bytes = (work["up_bytes"] + work["dn_bytes"]) * (w.blocks or 1)
    layer_roof = {"bytes_per_step": layer_bytes, "GBps": layer_bytes / (ms / 1e3) / 1e9,
                  "frac_hbm": layer_bytes / (ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                  "flops_per_step": (work["up_flops"] + work["dn_flops"]) * (w.blocks or 1)}
    layer_roof["TFLOPs"] = layer_roof["flops_per_step"] / (ms / 1e3) / 1e12
    layer_roof["frac_tensor"] = layer_roof["TFLOPs"] / peaks["bf16_tflops_sustained"]
    layer_roof["frac_tensor_of_burst"] = layer_roof["TFLOPs"] / peaks["bf16_tflops"]
    dn_ms = per_launch["down_proj"]
    layer_roof["down_proj"] = ({"GBps": work["dn_bytes"] / (dn_ms / 1e3) / 1e9,
                                "frac_hbm": work["dn_bytes"] / (dn_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                                "TFLOPs": work["dn_flops"] / (dn_ms / 1e3) / 1e12,
                                "frac_tensor": work["dn_flops"] / (dn_ms / 1e3) / 1e12 /
                                peaks["bf16_tflops_sustained"]} if dn_ms > 0 else None)
    rec["layer"] = layer_roof
    rec["kernel_ms"] = per_launch
    rec["experts_touched"] = n_touched
    rec["config"]["l2"] = "inputs larger than L2 (%.2f GB of weights per step)" % (layer_bytes / 1e9)
    rec["cpu_baseline"] = cpu_baseline(w, cpu_layers, inp, cpu_seconds) if with_cpu else None
    h.close()
    return rec, launches_per_step


def bench_ep(args, world, rank, dev):
    """Expert parallelism: rank r holds experts [r*E/N, (r+1)*E/N) of the one model and its own
    T tokens; a step is the whole layer on every rank, exchanges included (all-to-all over the
    default process group).  Needs torch.distributed (torchrun), any N that divides E."""
    import torch
    import torch.distributed as dist
    import moe_synth
    import mixture_experts_softmax_b200 as moe
    from mixture_experts_softmax_b200 import ep

    name = args.workload or "prefill"
    w = moe_synth.WORKLOADS[name]
    if w.blocks or w.bias is not None:
        raise SystemExit("--parallel ep runs the plain layer workloads (prefill, decode)")
    if not dist.is_initialized():
        raise SystemExit("--parallel ep needs torchrun (a process group), also for one GPU")
    ks, ws = default_steps(name)
    K = args.steps if args.steps is not None else ks
    W = max(3, args.warmup if args.warmup is not None else ws)
    full = moe_synth.make_inputs(w, device=dev).layers[0]          # the same model on every rank
    first, last = ep.expert_range(w.E, world, rank)
    rk = ep.EPRank(w.d, w.F, world, rank, ep.slice_experts(full, first, last), E=w.E, packed=args.layout == "packed")
    del full
    torch.cuda.empty_cache()
    x = moe_synth.draw_tokens(w.T, w.d, moe_synth.generator(w.seed + 1000 + rank, dev), dev)
    out = torch.empty_like(x)
    stream = torch.cuda.current_stream(dev)
    for _ in range(W):
        rk.forward(x, out)
    moe.check(moe.moe_sync_status(rk.layer.h, stream))
    R = int(max_over_ranks(args.repeats or 3, world, dev))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index) if rank == 0 else None
    if clocks:
        clocks.start()
    region_ms = []
    for r in range(R):
        barrier(world, dev)
        torch.cuda.synchronize(dev)
        if clocks and r == 0:
            clocks.mark("t0")
        e0.record(stream)
        for _ in range(K):
            rk.forward(x, out)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        region_ms.append(e0.elapsed_time(e1))
    if clocks:
        clocks.mark("t1")
    barrier(world, dev)
    clk = clocks.stop() if clocks else None
    moe.check(moe.moe_sync_status(rk.layer.h, stream))
    value, ms_max = job_value(w.T, world, statistics.median(region_ms) / K, dev)
    rk.close()
    return {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
            "repeats": R, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": DATA, "clocks": clk,
            "config": {"workload": name, "T_per_gpu": w.T, "d_model": w.d, "ffn": w.F, "experts": w.E,
                       "top_k": w.k, "parallelism": f"expert parallel x{world} ({w.E // world} experts per rank)",
                       "exchange": "torch.distributed all_to_all_single (counts, bf16 rows, fp32 results)",
                       "weights": "int8 + bf16 per-output-channel scales, layout " + args.layout}}


def run_native(args, world, rank, local):
    import torch
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if args.parallel == "ep":
        return bench_ep(args, world, rank, dev)
    head = args.workload or "prefill"
    with_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    rec, lps = bench_workload(head, args, world, rank, dev, args.layout, args.cpu_seconds, with_cpu)
    line = {"metric": METRIC, "value": rec["value"], "unit": "tokens/s", "n_gpus": world, "steps": rec["steps"],
            "warmup": rec["warmup"], "repeats": rec["repeats"], "ms_per_step": rec["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": DATA}
    line.update({k: v for k, v in rec.items() if k not in line and k not in ("unit",)})
    if lps is not None:
        line["gpu_launches"] = int(round(lps * rec["steps"]))
        line["gpu_launches_note"] = ("this library's kernel launches in one timed region of %d steps (%g per step; "
                                     "%d such regions were timed)" % (rec["steps"], lps, rec["repeats"]))
    # the other workloads, one process only (a multi-GPU run reports the headline workload)
    if args.workload is None and world == 1 and not (args.tokens or args.ffn):
        subs = {}
        for key, wname, layout in SUBRECORDS:
            import gc
            gc.collect()
            torch.cuda.empty_cache()
            # the API layout computes the same layer: its oracle baseline is the packed record's
            sub, slps = bench_workload(wname, argparse.Namespace(**{**vars(args), "steps": None, "warmup": None}),
                                       world, rank, dev, layout, SUB_CPU_SECONDS, with_cpu and layout == "packed")
            if slps is not None:
                sub["gpu_launches_per_step"] = slps
            subs[key] = sub
        line["workloads"] = subs
    return line


def kernel_times_over_regions(kernel_regions, K):
    """Per kernel, the median over the profiled regions of its mean launch time (ms), and the
    library's launches per step.  kernel_regions: one {kernel: (total ms, launches)} per region of
    K steps (moe_get_kernel_times after each region); a kernel that did not run reads 0."""
    names = list(kernel_regions[0])
    per_launch = {k: statistics.median([(kt[k][0] / kt[k][1] if kt[k][1] else 0.0) for kt in kernel_regions])
                  for k in names}
    launches_per_step = sum(n for _, n in kernel_regions[0].values()) / K
    return per_launch, launches_per_step


def cpu_baseline(w, cpu_layers, inp, budget_s):
    """The fp64 oracle on the host cores on a bounded sample of the same workload: the routing
    of the whole batch, then the expert FFNs of as many tokens as fit in the budget."""
    import oracle
    x = inp.x.cpu()
    cores = os.cpu_count()
    t_start = time.time()
    done = 0
    if w.blocks:
        gam = [{k: v.cpu() for k, v in g.items()} for g in inp.gammas]
        while done < x.shape[0] and (time.time() - t_start) < budget_s or done == 0:
            oracle.block_chain(cpu_layers, gam, x, eps=w.eps, tokens=[done])
            done += 1
        sample = f"{done} of {x.shape[0]} tokens through all {w.blocks} blocks"
    else:
        bias = None if inp.bias is None else inp.bias.cpu()
        oracle.route(x, cpu_layers[0]["router_w"], bias)   # routing of the whole batch
        while done < x.shape[0] and (time.time() - t_start) < budget_s or done == 0:
            oracle.forward(cpu_layers[0], x, bias=bias, tokens=[done])
            done += 1
        sample = f"routing of all {x.shape[0]} tokens + expert FFNs of {done} tokens"
    dt = time.time() - t_start
    return {"value": done / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample,
            "seconds": dt}


# ---- the reference arm: the CPU oracle ------------------------------------------------

def run_reference(args, world, rank):
    import moe_synth
    import oracle
    name = args.workload or "prefill"
    w = moe_synth.WORKLOADS[name]
    inp = moe_synth.make_inputs(w, device="cpu")
    K, W = args.steps, args.warmup
    x = inp.x
    bias = inp.bias
    per_step_tokens = 1

    def step(i):
        t = i % x.shape[0]
        if w.blocks:
            oracle.block_chain(inp.layers, inp.gammas, x, eps=w.eps, tokens=[t])
        else:
            oracle.forward(inp.layers[0], x, bias=bias, tokens=[t])

    for i in range(W):
        step(i)
    t0 = time.time()
    for i in range(K):
        step(W + i)
    dt = time.time() - t0
    value = K * per_step_tokens / dt
    cores = os.cpu_count()
    sample = f"{per_step_tokens} token of the {w.T}-token batch per step (expert FFNs of its 2 routes" + \
             (f", all {w.blocks} blocks" if w.blocks else "") + ")"
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": dt / K * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": DATA,
        "config": {"workload": name, "T_per_gpu": w.T, "d_model": w.d, "ffn": w.F, "experts": w.E,
                   "top_k": w.k, "blocks": w.blocks or 1},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return 0
        ks, ws = default_steps(args.workload or "prefill")
        args.steps = ks if args.steps is None else args.steps
        args.warmup = max(3, ws if args.warmup is None else args.warmup)
        if args.steps > 50 and args.workload != "tiny":
            args.steps = 20    # each step is about a second of fp64 work on the host
        line = run_reference(args, world, rank)
        print(json.dumps(line), flush=True)
        return 0
    world, rank, local = dist_setup(args.gpus)
    line = run_native(args, world, rank, local)
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist_teardown(world)
    return 0


if __name__ == "__main__":
    sys.exit(main())
