#!/usr/bin/env python
"""Benchmark of the dequantize-in-prologue quantized Linear on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
the pages' nn.Linear(3072, 4096) on x[32, 3072] in each weight-only format
(INT4 g128, NVFP4, MXFP4, FP8 E4M3 per-channel) plus the static-FP8 page's
two-layer 256->512->128 model on x[32, 256] -- six Linear layers, run as
four dqgemm_run calls and one dqgemm_run_static_mlp.  The metric is
microseconds per Linear layer (step time / 6), lower is better.

Weights rotate round-robin over R independent weight sets whose packed bytes
total at least 3x the L2 size, so every call streams its weight from HBM.
The timed region is K steps replayed as CUDA graphs (one graph per weight
set), bracketed by a barrier and a device synchronize, timed with CUDA
events; multi-GPU runs are independent replicas (no data-path collective)
and report the max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python bench.py --sweep        # M x (K, N) x format sweep, one JSON line per point
"""

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "DQ-GEMM µs/call; HBM GB/s (M≤128) & TFLOP/s (M≥1024) vs B200 roofline"
UNIT = "µs/call"
LIN_FORMATS = ("int4", "nvfp4", "mxfp4", "fp8")
# FP4 x FP4 (native block-scaled MMA, activations quantized per call): timed
# beside the step's formats at the same shape, not part of the step
W4A4_FORMATS = ("w4a4_mxfp4", "w4a4_nvfp4")
LM, LK, LN = 32, 3072, 4096
MLP_IN, MLP_HID, MLP_OUT = 256, 512, 128
CALLS_PER_STEP = len(LIN_FORMATS) + 2          # Linear layers (DQ-GEMMs) per step
LAUNCHES_PER_STEP = len(LIN_FORMATS) + 1       # the static MLP's two layers run in one launch
WORKLOAD = ("Linear(3072->4096), x[32,3072] bf16, in INT4-g128 / NVFP4 / MXFP4 / FP8-WO + "
            "static-FP8 MLP 256->512->128 (no bias), x[32,256]; 6 Linear layers per step in 5 launches "
            "(the MLP's two layers in one); value = step time / 6 layers")


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------


def algorithmic_bytes(fmt, M, K, N, bias=True):
    """Bytes one call must move: packed weight + scales (+ zero points, +
    global scale) + x + y + bias.  (W4A4: its weight storage format's bytes;
    the quantized activation is an intermediate, not an input.)"""
    fmt = {"w4a4_mxfp4": "mxfp4", "w4a4_nvfp4": "nvfp4"}.get(fmt, fmt)
    if fmt == "int4":
        w = N * K // 2 + N * (K // 128) * 2
    elif fmt == "int4_asym":
        w = N * K // 2 + N * (K // 128) * 3
    elif fmt == "nvfp4":
        w = N * K // 2 + N * (K // 16) + 4
    elif fmt == "mxfp4":
        w = N * K // 2 + N * (K // 32)
    elif fmt in ("fp8", "fp8_static"):
        w = N * K + N * 4
    else:
        raise ValueError(f"unknown format {fmt!r}")
    return w + M * K * 2 + M * N * 2 + (N * 2 if bias else 0)


# the sources that define the GEMM kernel itself (its launch parameters
# included); the other kernels and the host code do not change its traffic
GEMM_SOURCES = ("dq_common.cuh", "dq_gemm.cuh", "dq_layout.h")


def tensor_peak_ratio(fmt):
    """The format's dense tensor-core peak over bf16's (nominal 4.5 / 2.25
    PFLOP/s for FP8, 9 / 2.25 for FP4): the MMA each format runs."""
    return 2.0 if fmt == "fp8_static" else 4.0 if fmt in W4A4_FORMATS else 1.0


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "weight_only_quantized_prologue_b200", "csrc")
    for name in GEMM_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def ncu_traffic():
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken
    on the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("kernel_source_hash") != kernel_source_hash():
        return None
    return d.get("per_launch_bytes")


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling while the GPU is busy."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"dq_clocks_{os.getpid()}_{gpu_index}.csv")

    def start(self):
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            self.out.close()
            os.unlink(self.path)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        return parse_clock_samples(lines)


def parse_clock_samples(lines):
    """Median SM clock, max SM clock and the throttle reasons seen in
    `nvidia-smi --query-gpu=<ClockSampler.FIELDS> --format=csv,noheader,nounits`
    output lines; None when no line parses."""
    sm, mx, reasons = [], None, set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for line in lines:
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            mx = float(parts[2])
        except ValueError:
            continue
        for name, v in zip(names, parts[5:9]):
            if v.lower().startswith("active"):
                reasons.add(name)
    if not sm:
        return None
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# the workload on the GPU
# ---------------------------------------------------------------------------


class WeightSet:
    """One independent set of every layer of the step, packed on the GPU."""

    def __init__(self, idx, torch, dq, synthetic):
        self.layers = {}
        dev = "cuda"
        for j, fmt in enumerate(LIN_FORMATS):
            x, w, b = synthetic.linear_inputs(LM, LK, LN, seed=1000 * idx + j)
            self.layers[fmt] = dq.QuantizedLinear.from_float(fmt, w.to(dev), b.to(dev))
            if j == 0:
                self.x = x.to(dev)
        w1, w2 = synthetic.mlp_weights(seed=1000 * idx + 7)
        w1, w2 = w1.to(dev), w2.to(dev)
        # calibration: per-tensor min/max observers over ten seeded batches of
        # the float bf16 model (static FP8 page, "Calibrate, then insert ...")
        lo1 = hi1 = lo2 = hi2 = 0.0
        for s in range(1, 11):
            xc = synthetic.activations(LM, MLP_IN, seed=s).to(dev)
            hc = xc @ w1.t()
            lo1, hi1 = min(lo1, xc.min().item()), max(hi1, xc.max().item())
            lo2, hi2 = min(lo2, hc.min().item()), max(hi2, hc.max().item())
        s1 = float(torch.tensor(max(abs(lo1), abs(hi1)), dtype=torch.float32) / 448.0)
        s2 = float(torch.tensor(max(abs(lo2), abs(hi2)), dtype=torch.float32) / 448.0)
        self.mlp1 = dq.QuantizedLinear.from_float("fp8_static", w1.float(), None, act_scale=s1)
        self.mlp2 = dq.QuantizedLinear.from_float("fp8_static", w2.float(), None, act_scale=s2)
        self.xm = synthetic.activations(LM, MLP_IN, seed=1000 * idx + 8).to(dev)
        self.y = {f: torch.empty((LM, LN), dtype=torch.bfloat16, device=dev) for f in LIN_FORMATS}
        self.ym = torch.empty((LM, MLP_OUT), dtype=torch.bfloat16, device=dev)
        self.weight_bytes = sum(l.plan(LM)["weight_bytes"] for l in self.layers.values()) + \
            self.mlp1.plan(LM)["weight_bytes"] + self.mlp2.plan(LM)["weight_bytes"]

    def calls(self, dq, stream=None):
        """(name, launch) in step order: the four Linear layers, then the
        two-layer static MLP as one launch."""
        out = [(f, (lambda f=f: self.layers[f](self.x, out=self.y[f], stream=stream))) for f in LIN_FORMATS]
        out.append(("fp8_static_mlp", lambda: dq.static_mlp(self.mlp1, self.mlp2, self.xm, out=self.ym,
                                                             stream=stream)))
        return out

    def step(self, torch, dq, events=None):
        for i, (name, launch) in enumerate(self.calls(dq)):
            if events is not None:
                events[i][0].record()
            launch()
            if events is not None:
                events[i][1].record()


def run_ours(args, rank, world, local_rank):
    import torch

    import weight_only_quantized_prologue_b200 as dq
    from weight_only_quantized_prologue_b200 import synthetic

    torch.cuda.set_device(local_rank)
    props = torch.cuda.get_device_properties(local_rank)
    l2 = getattr(props, "L2_cache_size", 126 * 2**20)
    first = WeightSet(0, torch, dq, synthetic)
    R = max(2, math.ceil(3 * l2 / first.weight_bytes))
    sets = [first] + [WeightSet(i, torch, dq, synthetic) for i in range(1, R)]
    for s in sets:                       # first calls allocate split-K workspaces
        s.step(torch, dq)
    torch.cuda.synchronize()

    stream = torch.cuda.Stream()
    graphs = []
    with torch.cuda.stream(stream):
        for s in sets:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                s.step(torch, dq)
            graphs.append(g)
        # a second graph family with CUDA events around every call, for the
        # per-kernel durations behind the roofline figure
        n_ev = 2 * R
        ev = [[[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
               for _ in range(LAUNCHES_PER_STEP)]
              for _ in range(n_ev)]
        g_ev = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_ev, stream=stream):
            for i in range(n_ev):
                sets[i % R].step(torch, dq, events=ev[i])
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    sampler = ClockSampler(local_rank) if rank == 0 else None
    with torch.cuda.stream(stream):
        if sampler:
            sampler.start()
        settle_until = time.time() + args.settle_seconds   # clocks settle under load (untimed)
        i = 0
        while time.time() < settle_until:
            graphs[i % R].replay()
            i += 1
            if i % 200 == 0:
                stream.synchronize()
        for i in range(args.warmup):
            graphs[i % R].replay()
        stream.synchronize()
        barrier()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(args.steps):
            graphs[i % R].replay()
        t1.record(stream)
        t1.synchronize()
        torch.cuda.synchronize()
        barrier()
        ms_local = t0.elapsed_time(t1)
        clocks = sampler.stop() if sampler else None

        # per-kernel durations (events inside the graph)
        g_ev.replay()
        torch.cuda.synchronize()
    names = [c[0] for c in first.calls(dq)]
    per_call = {n: statistics.mean(ev[i][j][0].elapsed_time(ev[i][j][1]) for i in range(n_ev)) * 1000.0
                for j, n in enumerate(names)}

    ms = ms_local
    if world > 1:
        ms = aggregate_max(ms_local)

    # end-to-end through the public API with host buffers: per call, pinned
    # host x -> device, dqgemm_run, device y -> pinned host
    e2e_steps = max(3, min(args.steps, 200))
    e2e = EndToEnd(torch, dq, sets, stream)
    h2d, d2h = e2e.h2d_bytes, e2e.d2h_bytes
    e2e.run(3)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = e2e.run(e2e_steps, timed=True)
    e2e_ms = e0.elapsed_time(e1)
    if world > 1:
        e2e_ms = aggregate_max(e2e_ms)

    single = single_launch_us(torch, sets, stream)
    b2b, rotated_mb = {}, {}
    for f in LIN_FORMATS + W4A4_FORMATS:
        rot = FormatRotation(torch, dq, synthetic, f, l2)
        b2b[f] = back_to_back_us(torch, stream, rot.launches(stream))
        rotated_mb[f] = rot.rotated_mb
        rot.close()
    b2b_mlp = back_to_back_us(torch, stream, [
        (lambda st=st: dq.static_mlp(st.mlp1, st.mlp2, st.xm, out=st.ym, stream=stream)) for st in sets])
    wide = None if args.no_wide else wide_block(torch, dq, synthetic, stream, measured_peaks())

    for s in sets:
        for l in list(s.layers.values()) + [s.mlp1, s.mlp2]:
            assert l.last_error() == 0, "device-side wait timed out"

    value = job_us_per_call(ms, args.steps, CALLS_PER_STEP, world)
    peaks = measured_peaks()
    # the roofline kernel: the slowest weight-only format of the step, timed
    # as a stream of back-to-back calls of that format (the per-format figure
    # of the metric; a call's average duration in that stream)
    dom = max(LIN_FORMATS, key=b2b.get)
    alg = algorithmic_bytes(dom, LM, LK, LN)
    achieved = alg / (b2b[dom] * 1e-6) / 1e9
    traffic = ncu_traffic()
    roofline = {"bound": "hbm", "kernel": f"dq_gemm_kernel<{dom}, BN=32>", "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": (traffic or {}).get(dom), "algorithmic_bytes": alg,
                "avg_launch_us": round(b2b[dom], 3),
                "timing": (f"CUDA events around a graph of 240 back-to-back calls of this format, rotating "
                           f"over {rotated_mb[dom]} MB of distinct weights (>= 3x L2)"),
                "peak_source": f"{peaks['source']} (HBM copy)"}
    per_format = {}
    for n in LIN_FORMATS + W4A4_FORMATS:
        ab = algorithmic_bytes(n, LM, LK, LN)
        per_format[n] = {"us": round(b2b[n], 3), "GB/s": round(ab / (b2b[n] * 1e-6) / 1e9, 1),
                         "frac_hbm": round(ab / (b2b[n] * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
                         "rotated_MB": rotated_mb[n]}
        if n in per_call:
            per_format[n]["isolated_us"] = round(per_call[n], 3)
        else:
            per_format[n]["note"] = "FP4 x FP4, x quantized per call (2 or 3 launches); not in the step"
    per_format["fp8_static_mlp"] = {"us": round(b2b_mlp, 3), "isolated_us": round(per_call["fp8_static_mlp"], 3),
                                    "layers": 2}
    result = {
        "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 5), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": LM, "K": LK, "N": LN, "formats": list(LIN_FORMATS) + ["fp8_static"],
                   "weight_sets": R, "rotated_weight_MB": round(R * first.weight_bytes / 2**20, 1),
                   "l2_defeat": f"weights rotate over {R} sets >= 3x L2 ({l2 // 2**20} MB)",
                   "parallelism": f"replicas x{world}", "timing": "CUDA graphs, CUDA events"},
        "per_call": per_format,
        "roofline": roofline,
        "e2e": {"value": round(job_us_per_call(e2e_ms, e2e_steps, CALLS_PER_STEP, world), 4), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": args.steps * LAUNCHES_PER_STEP,
        "clocks": clocks,
        "single_launch_us": single,
        "wide": wide,
    }
    return result, sets


def back_to_back_us(torch, stream, launches, calls=240):
    """Device time per call of a list of launches run back to back (a CUDA
    graph of `calls` calls cycling over the list, as consecutive layers of a
    decode step run): the per-format figure of the metric.  Median of 5
    replays."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            for i in range(calls):
                launches[i % len(launches)]()
        g.replay()
        stream.synchronize()
        t = []
        for _ in range(5):
            a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            z.record(stream)
            z.synchronize()
            t.append(a.elapsed_time(z) * 1000.0 / calls)
    del g
    return statistics.median(t)


class FormatRotation:
    """One format's Linear at the page shape as many distinct copies of one
    packed weight as make >= 3x L2 (the back-to-back figure must not find
    its weights in L2), with one x and one y."""

    def __init__(self, torch, dq, synthetic, fmt, l2):
        import numpy as np

        x, w, b = synthetic.linear_inputs(LM, LK, LN, seed=4242)
        w = w.cuda()
        ps, pd, ss, sd = dq.storage_shapes(fmt, LK, LN)
        tdt = {np.uint8: torch.uint8, np.uint16: torch.int16, np.float32: torch.float32}
        packed = torch.empty(ps, dtype=tdt[pd], device="cuda")
        scales = torch.empty(ss, dtype=tdt[sd], device="cuda")
        g = dq.dqgemm_pack_device(fmt, w, packed, scales)
        bias = b.cuda()
        first = dq.QuantizedLinear(fmt, LK, LN, packed, scales, g, bias)
        wb = first.plan(LM)["weight_bytes"]
        R = max(2, math.ceil(3 * l2 / wb))
        self.layers = [first] + [dq.QuantizedLinear(fmt, LK, LN, packed, scales, g, bias) for _ in range(R - 1)]
        self.rotated_mb = round(R * wb / 2**20, 1)
        self.x = x.cuda()
        self.y = torch.empty((LM, LN), dtype=torch.bfloat16, device="cuda")
        for l in self.layers:               # first calls (W4A4: allocate the activation workspace)
            l(self.x, out=self.y)
        torch.cuda.synchronize()

    def launches(self, stream):
        return [(lambda l=l: l(self.x, out=self.y, stream=stream)) for l in self.layers]

    def close(self):
        for l in self.layers:
            assert l.last_error() == 0, "device-side wait timed out"
            l.close()
        self.layers = []


WIDE_M, WIDE_K, WIDE_N = 4096, 4096, 4096


def wide_block(torch, dq, synthetic, stream, peaks, reps=24):
    """The compute-bound half of the metric: M = K = N = 4096 per format,
    back-to-back calls alternating over 4 weight sets and 4 activation
    buffers (4 x (32 MB x + 32 MB y + weights) > L2); TFLOP/s counts the
    useful 2MKN.  Static FP8 includes its activation-quantize kernel."""
    out = {}
    M, K, N = WIDE_M, WIDE_K, WIDE_N
    xs = [synthetic.activations(M, K, seed=100 + i).cuda() for i in range(4)]
    ys = [torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for _ in range(4)]
    for fmt in list(LIN_FORMATS) + ["fp8_static"] + list(W4A4_FORMATS):
        layers = []
        for r in range(4):
            _, w, b = synthetic.linear_inputs(1, K, N, seed=200 + r)
            layers.append(dq.QuantizedLinear.from_float(fmt, w.cuda(), None if fmt == "fp8_static" else b.cuda(),
                                                        act_scale=0.011))
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            for i in range(4):
                layers[i](xs[i], out=ys[i], stream=stream)
            stream.synchronize()
            with torch.cuda.graph(g, stream=stream):
                for i in range(reps):
                    layers[i % 4](xs[i % 4], out=ys[i % 4], stream=stream)
            g.replay()
            stream.synchronize()
            t = []
            for _ in range(3):
                a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                g.replay()
                z.record(stream)
                z.synchronize()
                t.append(a.elapsed_time(z) * 1000.0 / reps)
        for l in layers:
            assert l.last_error() == 0, "device-side wait timed out"
        us = statistics.median(t)
        tflops = 2.0 * M * K * N / (us * 1e-6) / 1e12
        peak = peaks["bf16_tflops"] * tensor_peak_ratio(fmt)
        out[fmt] = {"us": round(us, 2), "TFLOP/s": round(tflops, 1), "frac_tensor": round(tflops / peak, 4),
                    "peak_tflops": round(peak, 1)}
        del g
        for l in layers:
            l.close()
    out["shape"] = {"M": M, "K": K, "N": N}
    out["peak_source"] = (f"{peaks['source']} bf16 dense (burst); FP8 = 2x and FP4 = 4x the bf16 figure "
                          "(the dense FP8:BF16 and FP4:BF16 ratios); static FP8 and W4A4 include their "
                          "activation-quantize kernels")
    return out


def single_launch_us(torch, sets, stream, reps=32):
    """Mean device time of one call on its own: the stream is idle apart
    from an L2 flush (a 256 MB memset) before it, so the call neither
    overlaps a neighbour nor finds its weight in L2.  Per weight-only format;
    None if the measurement itself fails (it is outside the timed step).
    (The event clock ticks about once a microsecond: single intervals are
    multiples of the tick, and a mean over many calls, whose starts fall at
    random phases of the tick, resolves below it.)"""
    try:
        flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        out = {}
        with torch.cuda.stream(stream):
            for f in LIN_FORMATS:
                lat = []
                for i in range(reps):
                    st = sets[i % len(sets)]
                    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    flush.zero_()
                    a.record(stream)
                    st.layers[f](st.x, out=st.y[f], stream=stream)
                    z.record(stream)
                    z.synchronize()
                    lat.append(a.elapsed_time(z) * 1000.0)
                out[f] = round(statistics.fmean(lat), 3)
        del flush
        return out
    except Exception as e:      # noqa: BLE001 - report, do not lose the bench line
        return {"error": str(e)[:200]}


class EndToEnd:
    """The step through the C ABI (its binding's dqgemm_run and
    dqgemm_run_static_mlp) with its data on the host: every step copies its
    inputs from pinned host memory (one packed copy) and its results back
    (one packed copy).  Uploads and downloads run on streams of
    their own over a ring of NB buffers, so later steps' inputs go up and
    earlier steps' results come down while step i computes; every byte of
    every step still crosses, inside the timed region."""

    NB = 2                                                        # buffers in flight (3 measured slower)
    IN = ("int4", "nvfp4", "mxfp4", "fp8", "fp8_static_l1")     # calls fed from the host
    OUT = ("int4", "nvfp4", "mxfp4", "fp8", "fp8_static_l2")    # results read back

    def __init__(self, torch, dq, sets, stream):
        self.torch, self.dq, self.sets, self.compute = torch, dq, sets, stream
        self.up, self.down = torch.cuda.Stream(), torch.cuda.Stream()
        self.cs = stream.cuda_stream              # the compute stream's handle, for the C calls
        s0 = sets[0]
        xs = {f: s0.x for f in LIN_FORMATS}
        xs["fp8_static_l1"] = s0.xm
        ys = {f: s0.y[f] for f in LIN_FORMATS}
        ys["fp8_static_l2"] = s0.ym
        self.in_shapes = [tuple(xs[n].shape) for n in self.IN]
        self.out_shapes = [tuple(ys[n].shape) for n in self.OUT]
        n_in = sum(a * b for a, b in self.in_shapes)
        n_out = sum(a * b for a, b in self.out_shapes)
        self.h2d_bytes, self.d2h_bytes = 2 * n_in, 2 * n_out
        bf = torch.bfloat16
        # host: each weight set's own inputs, packed; results per buffer
        self.h_in = []
        for st in sets:
            c = {f: st.x for f in LIN_FORMATS}
            c["fp8_static_l1"] = st.xm
            self.h_in.append(torch.cat([c[n].reshape(-1) for n in self.IN]).cpu().pin_memory())
        nb = self.NB
        self.h_out = [torch.empty(n_out, dtype=bf).pin_memory() for _ in range(nb)]
        self.d_in = [torch.empty(n_in, dtype=bf, device="cuda") for _ in range(nb)]
        self.d_out = [torch.empty(n_out, dtype=bf, device="cuda") for _ in range(nb)]
        # per-call operand addresses in each packed buffer, taken once
        self.vin = [{n: v.data_ptr() for n, v in zip(self.IN, self._views(self.d_in[b], self.in_shapes))}
                    for b in range(nb)]
        self.vout = [{n: v.data_ptr() for n, v in zip(self.OUT, self._views(self.d_out[b], self.out_shapes))}
                     for b in range(nb)]
        self.ev = {k: [torch.cuda.Event() for _ in range(nb)] for k in ("up", "done", "down")}

    @staticmethod
    def _views(flat, shapes):
        out, o = [], 0
        for a, b in shapes:
            out.append(flat[o:o + a * b].view(a, b))
            o += a * b
        return out

    def run(self, steps, timed=False):
        torch = self.torch
        e0 = e1 = None
        if timed:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(self.up)
        for i in range(steps):
            b, st = i % self.NB, self.sets[i % len(self.sets)]
            xin, yout = self.vin[b], self.vout[b]
            with torch.cuda.stream(self.up):
                if i >= self.NB:
                    self.up.wait_event(self.ev["done"][b])        # step i-NB has read d_in[b]
                self.d_in[b].copy_(self.h_in[i % len(self.sets)], non_blocking=True)
                self.ev["up"][b].record(self.up)
            # the calls name their stream; no stream context needed
            self.compute.wait_event(self.ev["up"][b])
            if i >= self.NB:
                self.compute.wait_event(self.ev["down"][b])       # step i-NB's results are home
            for f in LIN_FORMATS:
                self.dq.dqgemm_run(st.layers[f].handle, xin[f], LM, yout[f], self.cs)
            self.dq.dqgemm_run_static_mlp(st.mlp1.handle, st.mlp2.handle, xin["fp8_static_l1"], LM, None,
                                          yout["fp8_static_l2"], self.cs)
            self.ev["done"][b].record(self.compute)
            with torch.cuda.stream(self.down):
                self.down.wait_event(self.ev["done"][b])
                self.h_out[b].copy_(self.d_out[b], non_blocking=True)
                self.ev["down"][b].record(self.down)
        if timed:
            e1.record(self.down)          # after the last download, which follows all else
            e1.synchronize()
        else:
            self.down.synchronize()
        return e0, e1


def job_us_per_call(ms_max, steps, calls_per_step, world):
    """Whole-job time per call: every rank runs `steps` steps of
    `calls_per_step` calls; the job takes the slowest rank's time."""
    return ms_max * 1000.0 / (steps * calls_per_step * world)


def aggregate_max(v):
    """Max of a per-rank float over all ranks (the contract's device-time max)."""
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(v)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# the oracle on the host cores (cpu_baseline and --impl reference)
# ---------------------------------------------------------------------------


class OracleWorkload:
    """The same step computed by the fp64 oracle from its own packed storage
    (quantization itself is not timed: the GPU path also packs once)."""

    def __init__(self, synthetic):
        import numpy as np

        from oracle import linear as L

        self.L, self.np = L, np
        x, w, b = synthetic.linear_inputs(LM, LK, LN, seed=0)
        self.x = x.float().numpy().astype(np.float64)
        self.b = b.float().numpy().astype(np.float64)
        wv = w.numpy().astype(np.float64)
        self.store, self.pack_s = {}, {}
        for f in LIN_FORMATS:
            t0 = time.perf_counter()
            self.store[f] = L.quantize_pack(f, wv)
            self.pack_s[f] = time.perf_counter() - t0
        w1, w2 = synthetic.mlp_weights(seed=7)
        w1v, w2v = w1.float().numpy().astype(np.float64), w2.float().numpy().astype(np.float64)
        cal = [synthetic.activations(LM, MLP_IN, seed=s).float().numpy().astype(np.float64) for s in range(1, 11)]
        self.s1, self.s2 = L.calibrate_static_mlp(cal, w1v, w2v)
        self.q1 = L.quantize_pack("fp8", w1v)
        self.q2 = L.quantize_pack("fp8", w2v)
        self.xm = synthetic.activations(LM, MLP_IN, seed=8).float().numpy().astype(np.float64)
        from oracle.formats import bf16
        self.h = bf16(L.static_linear(L.quantize_act_fp8(self.xm, self.s1), self.s1,
                                      self.q1["packed"], self.q1["scales"]))

    def call(self, name, rows=None):
        """One call of the step; `rows` restricts the weight to its first
        `rows` output channels (a bounded sample of the call)."""
        L = self.L
        if name in LIN_FORMATS:
            st = self.store[name]
            p, s = st["packed"], st["scales"]
            if rows is not None:
                p, s = p[:rows], s[:rows]
            wd = L.dequant_exact(name, p, s, st["global_scale"])
            return L.linear_ref(self.x, wd, self.b[: wd.shape[0]])
        if name == "fp8_static_l1":
            p, s = self.q1["packed"], self.q1["scales"]
            return L.static_linear(L.quantize_act_fp8(self.xm, self.s1), self.s1, p[:rows], s[:rows])
        p, s = self.q2["packed"], self.q2["scales"]
        return L.static_linear(L.quantize_act_fp8(self.h, self.s2), self.s2, p[:rows], s[:rows])

    def rows_of(self, name):
        return {"fp8_static_l1": MLP_HID, "fp8_static_l2": MLP_OUT}.get(name, LN)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return len(os.sched_getaffinity(0))


def time_oracle_step(ow, fraction):
    """Seconds for one step of the oracle on `fraction` of each call's output
    channels, and the seconds scaled to the full step."""
    names = list(LIN_FORMATS) + ["fp8_static_l1", "fp8_static_l2"]
    t = 0.0
    for n in names:
        rows = max(16, int(ow.rows_of(n) * fraction) // 16 * 16)
        t0 = time.perf_counter()
        ow.call(n, rows=rows)
        t += (time.perf_counter() - t0) * ow.rows_of(n) / rows
    return t


def cpu_baseline(synthetic, budget_s=15.0):
    ow = OracleWorkload(synthetic)
    time_oracle_step(ow, 1.0 / 64)      # warm caches / BLAS
    t_full, n = 0.0, 0
    t_start = time.perf_counter()
    while n < 2 or time.perf_counter() - t_start < budget_s:
        t_full += time_oracle_step(ow, 1.0)
        n += 1
        if time.perf_counter() - t_start > 2 * budget_s:
            break
    us_per_call = t_full / n * 1e6 / CALLS_PER_STEP
    wall = time.perf_counter() - t_start
    # the same step on one BLAS thread, on a bounded share of every call's
    # output channels (about 5 s), scaled to the full step
    single = None
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1, user_api="blas"):
            probe = time_oracle_step(ow, 1.0 / 64)
            frac = min(1.0, max(1.0 / 64, 5.0 / max(probe, 1e-9)))
            single = round(time_oracle_step(ow, frac) * 1e6 / CALLS_PER_STEP, 1)
    except ImportError:
        pass
    return {"value": round(us_per_call, 1), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} full oracle steps (6 calls each: dequantize-exact + fp64 GEMM, "
                      f"storage packed beforehand), {wall:.1f} s",
            "single_core_value": single,
            "quantize_pack_s": {f: round(v, 3) for f, v in ow.pack_s.items()}}


def run_reference(args, rank, world):
    from weight_only_quantized_prologue_b200 import synthetic

    if rank != 0:
        return None
    ow = OracleWorkload(synthetic)
    # size each step so that warmup + steps end within ~2 minutes
    probe = time_oracle_step(ow, 1.0 / 64)
    per_step_budget = 120.0 / max(1, args.steps + args.warmup)
    fraction = min(1.0, max(1.0 / 256, per_step_budget / max(probe, 1e-9)))
    for _ in range(args.warmup):
        time_oracle_step(ow, fraction)
    t0 = time.perf_counter()
    scaled = 0.0
    for _ in range(args.steps):
        scaled += time_oracle_step(ow, fraction)
    wall = time.perf_counter() - t0
    value = scaled * 1e6 / (args.steps * CALLS_PER_STEP)
    sample = (f"each step computes {fraction:.4g} of every call's output channels with the fp64 oracle "
              f"(dequantize-exact + GEMM) and scales its time to the full call; {wall:.1f} s total")
    return {"metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(scaled * 1000.0 / args.steps, 3),
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD, "M": LM, "K": LK, "N": LN,
                       "formats": list(LIN_FORMATS) + ["fp8_static"], "parallelism": "host cores"},
            "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------------------
# sweep (M x (K, N) x format), one JSON line per point
# ---------------------------------------------------------------------------


def run_ncu_case(fmt, M=LM, K=LK, N=LN):
    """Eight back-to-back calls of one format, rotating over four weight
    sets: the case the committed ncu captures take (one launch, after four
    warm ones).  Default shape: the step's Linear at M=32."""
    import torch

    import weight_only_quantized_prologue_b200 as dq
    from weight_only_quantized_prologue_b200 import synthetic

    torch.cuda.set_device(0)
    layers = []
    for r in range(4):
        _, w, b = synthetic.linear_inputs(1, K, N, seed=r)
        layers.append(dq.QuantizedLinear.from_float(fmt, w.cuda(), None if fmt == "fp8_static" else b.cuda(),
                                                    act_scale=0.011))
    xc = synthetic.activations(M, K, seed=1).cuda()
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    for i in range(8):
        layers[i % 4](xc, out=y)
    torch.cuda.synchronize()
    for l in layers:
        assert l.last_error() == 0, "device-side wait timed out"
    print(json.dumps({"ncu_case": fmt, "M": M, "K": K, "N": N, "plan": layers[0].plan(M)}), flush=True)


def run_sweep(args):
    import torch

    import weight_only_quantized_prologue_b200 as dq
    from weight_only_quantized_prologue_b200 import synthetic

    torch.cuda.set_device(0)
    peaks = measured_peaks()
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    Ms = [int(m) for m in args.sweep_m.split(",")]
    shapes = [tuple(int(v) for v in s.split("x")) for s in args.sweep_kn.split(",")]
    fmts = args.sweep_formats.split(",")
    for (K, N) in shapes:
        for fmt in fmts:
            wb = algorithmic_bytes(fmt, 0, K, N, bias=False)
            R = max(2, math.ceil(3 * l2 / wb))
            layers = []
            for r in range(R):
                _, w, b = synthetic.linear_inputs(1, K, N, seed=r)
                layers.append(dq.QuantizedLinear.from_float(fmt, w.cuda(), None if fmt == "fp8_static" else b.cuda(),
                                                            act_scale=0.02))
            for M in Ms:
                x = synthetic.activations(M, K, seed=1).cuda()
                y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
                for l in layers:
                    l(x, out=y)
                torch.cuda.synchronize()
                flops = 2.0 * M * K * N
                reps = max(R, min(400, int(2e11 / max(flops, 1))))
                stream = torch.cuda.Stream()
                with torch.cuda.stream(stream):
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=stream):
                        for i in range(reps):
                            layers[i % R](x, out=y)
                    g.replay()
                    stream.synchronize()
                    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    t0.record(stream)
                    g.replay()
                    t1.record(stream)
                    t1.synchronize()
                us = t0.elapsed_time(t1) * 1000.0 / reps
                for l in layers:
                    # a timed-out call wrote nothing: its time is no measurement
                    assert l.last_error() == 0, f"device-side wait timed out: {fmt} {M}x{K}x{N}"
                byts = algorithmic_bytes(fmt, M, K, N, bias=fmt != "fp8_static")
                gbs = byts / (us * 1e-6) / 1e9
                tflops = flops / (us * 1e-6) / 1e12
                peak_t = peaks["bf16_tflops"] * tensor_peak_ratio(fmt)
                print(json.dumps({"fmt": fmt, "M": M, "K": K, "N": N, "us": round(us, 3),
                                  "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
                                  "TFLOP/s": round(tflops, 1), "frac_tensor": round(tflops / peak_t, 4),
                                  "plan": layers[0].plan(M)}), flush=True)
                del g
            for l in layers:
                l.close()


# ---------------------------------------------------------------------------


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-wide", action="store_true", help="skip the M=4096 compute-bound block")
    ap.add_argument("--settle-seconds", type=float, default=1.5,
                    help="untimed load before the warmup so clocks settle and get sampled")
    ap.add_argument("--sweep", action="store_true")
    ap.add_argument("--sweep-m", default="1,16,32,128,1024,4096")
    ap.add_argument("--sweep-kn", default="4096x4096,4096x14336,14336x4096")
    ap.add_argument("--sweep-formats", default="int4,nvfp4,mxfp4,fp8,fp8_static")
    ap.add_argument("--ncu-case", choices=list(LIN_FORMATS) + ["fp8_static", "int4_asym"] + list(W4A4_FORMATS),
                    default=None,
                    help="small profiling case: 8 plain launches of one format (4 weight sets, no graphs, "
                         "no timing) for an ncu capture; the step's shape unless --ncu-shape is given")
    ap.add_argument("--ncu-shape", default=None, help="MxKxN of the profiling case, e.g. 4096x4096x4096")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.sweep:
        run_sweep(args)
        return
    if args.ncu_case:
        shape = [int(v) for v in args.ncu_shape.split("x")] if args.ncu_shape else [LM, LK, LN]
        run_ncu_case(args.ncu_case, *shape)
        return

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    res, sets = run_ours(args, rank, world, local_rank)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            from weight_only_quantized_prologue_b200 import synthetic
            res["cpu_baseline"] = cpu_baseline(synthetic)
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
