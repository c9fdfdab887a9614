#!/usr/bin/env python
"""Benchmark of the NVFP4 dense SwiGLU FFN on B200.

One step = one FFN layer forward (fused gate+up projection with the SiLU*mul
epilogue, then the down projection) over one batch of the workload's
synthetic input, through the library's C ABI.  Default workload: prefill,
m=4096 rows, hidden 5120, inter 17408, bf16 activations (W4A16); the value is
whole-job TFLOP/s (2 * m * 3 * hidden * inter flops per step).  The same run
also times the m=1 decode layer (weight GB/s) and the fixed-format W4A4 layer,
reported as sub-objects.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
       [--workload prefill|decode|smallm|w4a4] [--m M] [--no-extra] [--no-cpu]
Under torchrun each rank runs its own replica (the FFN has no cross-GPU step
here): the timed region is bracketed by a barrier and a device synchronise,
the time is the max over ranks, and the value sums all ranks' work.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 FFN µs/layer & TFLOP/s (m=4096); weight GB/s (m=1) vs roofline"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

WORKLOADS = {
    # name: (synth recipe, m, hidden, inter, activation format)
    "prefill": ("prefill", 4096, 5120, 17408, "bf16"),
    "decode": ("decode", 1, 5120, 17408, "bf16"),
    "smallm": ("smallm", 64, 5120, 17408, "bf16"),
    "w4a4": ("w4a4", 512, 4096, 12288, "nvfp4_fixed"),
}


def max_over_ranks(value: float, dist, device) -> float:
    """Max of a per-rank scalar (a time) over all ranks; identity without a group."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(units_per_step: float, steps: int, max_ms: float, world: int) -> float:
    """Whole-job throughput: every rank did `steps` steps of `units_per_step`
    units; the job took the slowest rank's time."""
    return world * units_per_step * steps / (max_ms * 1e-3)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# Nominal dense FP4 / bf16 tensor-core throughput ratio (9 vs 2.25 PFLOP/s),
# used only when the library's own block-scaled FP4 MMA probe could not run.
FP4_OVER_BF16 = 4.0


def tensor_peak(peaks, fmt):
    """(TFLOP/s, description) of the tensor-core peak for a projection's dtype:
    the measured bf16 matmul peak, and for the fixed format the measured
    kind::mxf4nvf4 probe ('fp4_tflops', added at run time) when present."""
    if fmt == "nvfp4_fixed":
        if peaks.get("fp4_tflops"):
            return peaks["fp4_tflops"], "fp4 (tcgen05 kind::mxf4nvf4 probe, measured in this run)"
        return peaks["bf16_tflops"] * FP4_OVER_BF16, "bf16 x nominal fp4/bf16 ratio 4"
    return peaks["bf16_tflops"], "bf16"


def measure_tensor_probes(native):
    """Dense tensor-core TFLOP/s of this GPU for the MMA kinds the library
    issues (its own probe kernels; best of one and two issuing threads)."""
    out = {}
    for kind in ("bf16", "nvfp4"):
        try:
            out[kind] = round(max(native.ffn_nvfp4_tensor_peak(kind, issuers, 20000) for issuers in (1, 2)), 1)
        except Exception as e:  # reported, never fatal to the bench line
            out[kind] = None
            out[kind + "_error"] = str(e)
    return out


def ffn_flops(m, H, I):
    return 2.0 * m * 3 * H * I


def nvfp4_bytes(n, k):
    return n * k / 2 + n * k / 16


# --------------------------------------------------------------- clocks

# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# one ncu capture, keyed by (kernel, workload, m), with a fingerprint of the kernel
# sources it was taken on (comments and whitespace ignored): reported only
# while the sources are unchanged.
KERNEL_SOURCES = ("csrc/tc_gemm.cu", "csrc/sm100.cuh", "csrc/common.cuh", "csrc/internal.h")
TRAFFIC = {
    ("tc_w4a16_gate_up_silu", "prefill", 4096): {
        "bytes": 147362560 + 128156160, "sources_sha1": "1bcc724ab03551f65ac0366f5525c5aca1bb4146"},
    ("tc_planes_layer", "decode", 1): {
        "bytes": 150511872 + 3119872, "sources_sha1": "1bcc724ab03551f65ac0366f5525c5aca1bb4146"},
    ("tc_w4a4_gate_up_silu_quant", "w4a4", 512): {
        "bytes": 57844736 + 466944, "sources_sha1": "1bcc724ab03551f65ac0366f5525c5aca1bb4146"},
    ("tc_w4a4_gate_up_silu_quant", "w4a4", 1): {
        "bytes": 56699904 + 512, "sources_sha1": "1bcc724ab03551f65ac0366f5525c5aca1bb4146"},
}


def normalised_source(text):
    """Source text without comments and whitespace (edits to either do not
    change the compiled kernel)."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return re.sub(r"\s+", "", text)


def kernel_sources_sha1(read=None):
    import hashlib
    pkg = os.path.join(os.path.dirname(os.path.abspath(__file__)), "nvfp4_quantized_dense_w4a16_b200")
    if read is None:
        def read(rel):
            with open(os.path.join(pkg, rel), encoding="utf-8") as fh:
                return fh.read()
    h = hashlib.sha1()
    for f in KERNEL_SOURCES:
        h.update(normalised_source(read(f)).encode())
    return h.hexdigest()


def measured_traffic(kname, workload, m=None):
    t = TRAFFIC.get((kname, workload, m))
    if t is None or t["sources_sha1"] != kernel_sources_sha1():
        return None
    return t["bytes"]


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    @staticmethod
    def _die_with_parent():
        # the sampler must not outlive this process, even if it crashes
        # (a profiler waits for every process of the tree to exit)
        import ctypes
        import signal
        ctypes.CDLL("libc.so.6", use_errno=True).prctl(1, signal.SIGTERM)  # PR_SET_PDEATHSIG

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.tmp, stderr=subprocess.DEVNULL, preexec_fn=self._die_with_parent)
        except OSError:
            self.proc = None
        if self.proc is not None:
            import atexit
            atexit.register(self.proc.kill)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        self.tmp.seek(0)
        rows = [r.split(",") for r in self.tmp.read().strip().splitlines() if r.strip()]
        os.unlink(self.tmp.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except (ValueError, IndexError):
                continue
            for nm, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------- our arm

class Workload:
    def __init__(self, native, name, m=None):
        import torch
        from nvfp4_quantized_dense_w4a16_b200 import synth
        recipe, m0, H, I, fmt = WORKLOADS[name]
        self.name, self.m, self.H, self.I, self.fmt = name, (m or m0), H, I, fmt
        inp = synth.make_inputs(recipe, m=self.m)
        dev = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).cuda()
        q = []
        for bits in (inp.w_gate, inp.w_up, inp.w_down):
            w = dev(bits)
            q.append(native.ffn_nvfp4_quantize_weights(w))
            del w
        self.weight_bytes = nvfp4_bytes(2 * I, H) + nvfp4_bytes(H, I)
        # weight layouts the handles hold: the few-row bf16 workloads also keep
        # the natural tiles, which the block-scaled FP4 path for m <= 8 streams
        self.layouts = "all" if (fmt == "bf16" and name in ("decode", "smallm")) else fmt
        # A step that reads less than twice the L2 would find part of its
        # weights still cached from earlier steps: such layers rotate through R
        # copies of their weights (R x weight bytes >= 4 x L2), so every step
        # streams weights that 3+ other steps' worth of traffic has evicted.
        act_bytes = self.m * (H + I) * 2 * 2
        self.sets = 1
        if self.weight_bytes + act_bytes < 2 * L2_BYTES:
            self.sets = int(math.ceil(4 * L2_BYTES / self.weight_bytes))
        self.handles = []
        for _ in range(self.sets):
            g, u, d = (native.ffn_nvfp4_weight_create(*t, formats=self.layouts) for t in q)
            self.handles.append((native.ffn_nvfp4_weight_create_gate_up(g, u), d))
            del g, u
        del q
        self.gate_up, self.down = self.handles[0]
        self.x = dev(inp.x)
        self.x_bits = inp.x
        self.out = torch.empty((self.m, H), dtype=torch.bfloat16, device="cuda")
        self.ws = torch.empty((max(16, native.ffn_nvfp4_workspace_size(self.m, H, I, fmt)),),
                              dtype=torch.uint8, device="cuda")
        self.native = native
        torch.cuda.synchronize()
        self.flush_l2 = False
        self.l2_note = (f"weights rotated through {self.sets} copies ({self.sets} x "
                        f"{self.weight_bytes / 1e6:.1f} MB >= 4 x L2)" if self.sets > 1
                        else "reads per step exceed 2 x L2")

    def step(self, i=0):
        gate_up, down = self.handles[i % self.sets]
        self.native.ffn_nvfp4_forward(self.x, gate_up, down, self.fmt, out=self.out, workspace=self.ws)

    def kernel_units(self, kname, peaks):
        """(bound, algorithmic flops or bytes per launch) of a kernel of this layer."""
        m, H, I = self.m, self.H, self.I
        if "quantize_activations" in kname:
            return "hbm", None
        if "planes_prologue" in kname:  # reads x (its planes are a few KB)
            return "hbm", m * H * 2
        if "planes_layer" in kname:  # both projections in one persistent kernel
            return "hbm", self.weight_bytes + m * H * 2 * 2 + m * I * 2 * 2
        if "gate_up" in kname:
            flops, byts = 2.0 * m * 2 * I * H, nvfp4_bytes(2 * I, H) + m * H * 2 + m * I * 2
        else:
            flops, byts = 2.0 * m * H * I, nvfp4_bytes(H, I) + m * I * 2 + m * H * 2
        # tensor-bound when the arithmetic intensity exceeds the ridge point of
        # the projection's own tensor peak
        ridge = tensor_peak(peaks, self.fmt)[0] * 1e12 / (peaks["hbm_gbs"] * 1e9)
        return ("tensor", flops) if flops / byts > ridge else ("hbm", byts)


def roofline(wl, prof, peaks, peak_src, workload):
    """The `roofline` object for the dominant kernel of a profile
    {kernel name: (launches, total ms)}: algorithmic units per launch over the
    average launch duration, against the peak of the bound it is under."""
    if not prof:
        return None
    # the longest kernel whose algorithmic units are known
    ranked = sorted(prof.items(), key=lambda kv: -kv[1][1])
    known = [kv for kv in ranked if wl.kernel_units(kv[0], peaks)[1] is not None]
    kname, (launches, kms) = (known or ranked)[0]
    bound, units = wl.kernel_units(kname, peaks)
    if units is None:
        return None
    avg_s = kms / launches * 1e-3
    if bound == "tensor":
        peak, what = tensor_peak(peaks, wl.fmt)
        achieved = units / avg_s / 1e12
        unit = "TFLOP/s"
    else:
        peak, what = peaks["hbm_gbs"], "HBM copy"
        achieved = units / avg_s / 1e9
        unit = "GB/s"
    return {"kernel": kname, "bound": bound, "achieved": round(achieved, 2), "peak": peak,
            "peak_source": f"{peak_src} ({what})", "unit": unit, "frac": round(achieved / peak, 4),
            "traffic": measured_traffic(kname, workload, wl.m),
            "avg_launch_us": round(avg_s * 1e6, 2), "launches": launches}


def run_ours(args, rank, world, dist):
    import torch
    from nvfp4_quantized_dense_w4a16_b200 import build as B
    B.build()
    from nvfp4_quantized_dense_w4a16_b200 import native as N

    peaks, peak_src = load_peaks()
    dev_index = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(dev_index)
    probes = measure_tensor_probes(N)
    if probes.get("nvfp4"):
        peaks["fp4_tflops"] = probes["nvfp4"]
    wl = Workload(N, args.workload, args.m)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda") if wl.flush_l2 else None

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    clocks = Clocks(dev_index)
    clocks.start()
    for i in range(args.warmup):
        wl.step(i)
    barrier()
    ms_local, prof = time_steps(N, wl, args.steps, flush, args.eager, barrier)
    ms = max_over_ranks(ms_local, dist, "cuda")
    clk = clocks.stop()
    ms_step = ms / args.steps
    flops = ffn_flops(wl.m, wl.H, wl.I)
    value = aggregate_throughput(flops, args.steps, ms, world) / 1e12

    roof = roofline(wl, prof, peaks, peak_src, args.workload)
    kernels = {k: {"launches": l, "total_ms": round(t, 4), "share": round(t / max(1e-9, sum(v[1] for v in prof.values())), 4)}
               for k, (l, t) in prof.items()}
    gpu_launches = sum(v[0] for v in prof.values())

    # end to end through the public API with pinned host buffers
    x_host = torch.from_numpy(np.ascontiguousarray(wl.x_bits).view(np.int16)).view(torch.bfloat16).pin_memory()
    out_host = torch.empty((wl.m, wl.H), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(wl.x)
    e2e_steps = max(3, min(args.steps, 50))
    for _ in range(2):
        x_dev.copy_(x_host, non_blocking=True)
        N.ffn_nvfp4_forward(x_dev, wl.gate_up, wl.down, wl.fmt, out=wl.out, workspace=wl.ws)
        out_host.copy_(wl.out, non_blocking=True)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(e2e_steps):
        x_dev.copy_(x_host, non_blocking=True)
        gate_up, down = wl.handles[i % wl.sets]
        N.ffn_nvfp4_forward(x_dev, gate_up, down, wl.fmt, out=wl.out, workspace=wl.ws)
        out_host.copy_(wl.out, non_blocking=True)
    e1.record()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, "cuda")
    e2e = {"value": round(aggregate_throughput(flops, e2e_steps, e2e_ms, world) / 1e12, 3), "unit": "TFLOP/s",
           "h2d_bytes_per_step": wl.m * wl.H * 2, "d2h_bytes_per_step": wl.m * wl.H * 2,
           "ms_per_step": round(e2e_ms / e2e_steps, 4)}

    l2_note, layouts = wl.l2_note, wl.layouts
    extra = {}
    if not args.no_extra and args.workload == "prefill":
        del wl, x_dev
        torch.cuda.empty_cache()
        extra["decode_m1"] = secondary(N, "decode", [1], peaks, max(args.steps, 20), args.eager)[1]
        extra["smallm"] = secondary(N, "smallm", [8, 16, 32, 64], peaks, max(args.steps, 20), args.eager)
        w4 = secondary(N, "w4a4", [1, 7, 64, 512], peaks, max(args.steps // 2, 10), args.eager)
        extra["w4a4_m512"] = w4.pop(512)
        extra["w4a4_small"] = w4
        torch.cuda.empty_cache()
    extra["tensor_probes_tflops"] = probes
    return {
        "value": round(value, 3), "ms_per_step": round(ms_step, 4), "roofline": roof,
        "kernels": kernels, "gpu_launches": gpu_launches, "clocks": clk, "e2e": e2e,
        "workload": args.workload, "m": args.m or WORKLOADS[args.workload][1], "extra": extra,
        "l2": l2_note, "layouts": layouts,
    }


def time_steps(N, wl, steps, flush, eager, barrier):
    """Time `steps` forward steps; returns (total ms, per-kernel profile).

    Default: the steps are captured in one CUDA graph with a timing-event pair
    around each step, replayed once untimed and once timed; per-kernel
    durations come from launching the same steps directly with an event pair
    around every kernel (events between kernels also keep them from
    overlapping, which is why the timed graph has none).  With `eager` (for
    runs under a profiler) the steps are launched directly and timed with the
    same events, which then include host launch latency."""
    import torch
    if eager:
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        stops = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        N.ffn_nvfp4_profile_begin()
        for i in range(steps):
            if flush is not None:
                flush.zero_()
            starts[i].record()
            wl.step(i)
            stops[i].record()
        barrier()
        prof = N.ffn_nvfp4_profile_end()
        return sum(a.elapsed_time(b) for a, b in zip(starts, stops)), prof
    graph, starts, stops = capture_steps(N, wl, steps, flush)
    graph.replay()  # untimed: loads the graph onto the device
    barrier()
    graph.replay()  # the timed region
    barrier()
    ms = sum(a.elapsed_time(b) for a, b in zip(starts, stops))
    del graph
    # per-kernel durations: the same steps launched directly with an event
    # pair around every kernel (recorded on the stream in front of and behind
    # each launch, so each pair brackets that kernel's own execution)
    N.ffn_nvfp4_profile_begin()
    for i in range(steps):
        if flush is not None:
            flush.zero_()
        wl.step(i)
    barrier()
    prof = N.ffn_nvfp4_profile_end()
    return ms, prof


def capture_steps(N, wl, steps, flush):
    """Capture `steps` forward steps (each after an optional L2 flush, between
    a pair of timing events) into one CUDA graph, so every timestamp is taken
    on the device during replay and none includes host launch latency.
    Returns (graph, starts, stops)."""
    import torch
    starts = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(steps)]
    stops = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(steps)]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=torch.cuda.Stream()):
        for i in range(steps):
            if flush is not None:
                flush.zero_()
            starts[i].record()
            wl.step(i)
            stops[i].record()
    return graph, starts, stops


def secondary(N, name, ms, peaks, steps, eager=False):
    """Time other layer shapes of one workload (its weights built once) at
    each row count in `ms`: {m: per-step µs, weight GB/s, TFLOP/s, fraction
    of the roofline, per-kernel µs}."""
    import torch
    wl = Workload(N, name, max(ms))
    x_all, out_all = wl.x, wl.out
    res = {}
    for m in ms:
        wl.m, wl.x, wl.out = m, x_all[:m].contiguous(), out_all[:m]
        wl.ws = torch.empty((max(16, N.ffn_nvfp4_workspace_size(m, wl.H, wl.I, wl.fmt)),), dtype=torch.uint8,
                            device="cuda")
        for i in range(3):
            wl.step(i)
        torch.cuda.synchronize()
        ms_total, prof = time_steps(N, wl, steps, None, eager, torch.cuda.synchronize)
        t = ms_total / steps * 1e-3
        byts = wl.weight_bytes + m * (wl.H + wl.I) * 2 * 2
        flops = ffn_flops(m, wl.H, wl.I)
        roof = max(byts / (peaks["hbm_gbs"] * 1e9), flops / (tensor_peak(peaks, wl.fmt)[0] * 1e12))
        res[m] = {"m": m, "hidden": wl.H, "inter": wl.I, "format": wl.fmt, "us_per_layer": round(t * 1e6, 2),
                  "weight_gbs": round(wl.weight_bytes / t / 1e9, 1),
                  "tflops": round(flops / t / 1e12, 3),
                  "hbm_roofline_frac": round(wl.weight_bytes / t / 1e9 / peaks["hbm_gbs"], 4),
                  "roofline_frac": round(roof / t, 4),
                  "kernels": {k: {"launches": l, "avg_us": round(tt / l * 1e3, 2)} for k, (l, tt) in prof.items()}}
    del wl
    return res


# --------------------------------------------------------------- CPU oracle

def oracle_sample(name, rows, reps, warmup=0):
    """Time the CPU oracle on `rows` rows of the workload (after quantising the
    weights with the oracle).  Returns (seconds per rep, flops per rep, threads)."""
    from nvfp4_quantized_dense_w4a16_b200 import synth
    from oracle import nvfp4_ffn as O
    recipe, m0, H, I, fmt = WORKLOADS[name]
    inp = synth.make_inputs(recipe, m=max(rows, 1))
    q = [O.quantize_weight(synth.bf16_bits_to_f32(b)) for b in (inp.w_gate, inp.w_up, inp.w_down)]
    x = synth.bf16_bits_to_f32(inp.x[:rows]).astype(np.float64)
    f = O.ffn_w4a16 if fmt == "bf16" else O.ffn_w4a4
    for _ in range(warmup):
        f(x, *q)
    times = []
    for _ in range(reps):
        t0 = time.perf_counter()
        f(x, *q)
        times.append(time.perf_counter() - t0)
    try:
        from threadpoolctl import threadpool_info
        threads = max([p.get("num_threads", 1) for p in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count() or 1
    return times, ffn_flops(rows, H, I), threads


def cpu_baseline(name, rows=1, reps=1):
    times, fl, threads = oracle_sample(name, rows, reps)
    s = statistics.mean(times)
    return {"value": round(fl / s / 1e12, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{rows} row(s) of the {name} workload through the fp64 numpy oracle "
                      f"(weights pre-quantised by the oracle), mean of {reps} run(s), {s:.2f} s each"}


def run_reference(args):
    rows = 1
    times, fl, threads = oracle_sample(args.workload, rows, args.steps, warmup=min(args.warmup, 1))
    s = sum(times)
    value = fl * args.steps / s / 1e12
    recipe, m0, H, I, fmt = WORKLOADS[args.workload]
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(s / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "m": args.m or m0, "hidden": H, "inter": I,
                   "act_format": fmt, "sample_rows_per_step": rows},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"{rows} row per step of the {args.workload} workload (fp64 numpy oracle)"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="prefill")
    ap.add_argument("--m", type=int, default=None)
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="launch the timed steps directly instead of through a CUDA graph "
                         "(for runs under a profiler; times then include launch latency)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            run_reference(args)
        return

    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    res = run_ours(args, rank, world, dist)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    recipe, m0, H, I, fmt = WORKLOADS[args.workload]
    cpu = None
    if world == 1 and not args.no_cpu:
        cpu = cpu_baseline(args.workload)
    line = {
        "metric": METRIC, "value": res["value"], "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
        "us_per_layer": round(res["ms_per_step"] * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 x nvfp4 (fp32 accumulate)" if fmt == "bf16" else "nvfp4 x nvfp4 (fp32 accumulate)",
        "data": "synthetic (seeded numpy draws; random-init weights)",
        "config": {"workload": args.workload, "m": res["m"], "hidden": H, "inter": I, "act_format": fmt,
                   "parallelism": f"replicas x{world}", "l2": res["l2"], "weight_layouts": res["layouts"],
                   "launch": ("eager launches" if args.eager else
                              "the K timed steps captured in one CUDA graph, replayed once; "
                              "kernel durations from the same steps launched directly with an event "
                              "pair per kernel")},
        "roofline": res["roofline"], "cpu_baseline": cpu, "e2e": res["e2e"],
        "gpu_launches": res["gpu_launches"], "kernels": res["kernels"], "clocks": res["clocks"],
    }
    line.update(res["extra"])
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
