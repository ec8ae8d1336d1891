#!/usr/bin/env python
"""Benchmark of the fused W4A4 + low-rank linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl twq|reference]

One step is one pass of the hot path over one batch on inputs already resident
in HBM: BF16 X to BF16 Y through the online activation quantizer and the fused
dual-component layer. For decode batches (b <= 16) that is one launch of
twq_fused_linear_x, which quantizes X inside the layer kernel; otherwise it is
twq_quantize_act_i8 followed by twq_fused_linear_i8 (the 4-bit codes stored one
per byte). The step on packed codes (twq_quantize_act + twq_fused_linear) is timed
beside it. The default workload is the large MLP layer (b = 8192, m = 5120,
n = 25600, r = 256), the largest that fits one GPU. Steps run from a CUDA
graph on one stream; the K timed steps are bracketed by a barrier and a device
synchronize, timed with CUDA events, max over ranks. Packed weights rotate over
enough copies that consecutive uses of one copy are more than 2x the 126 MB L2
apart, so weight bytes come from HBM.

Multi-GPU: the layer shards over tokens with replicated weights and no data
exchange (replicas), so each rank runs the same per-GPU workload ("weak").

Prints one JSON line. With --impl reference the CPU oracle is timed on the host
cores instead, on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
INT8_PER_BF16 = 2.0  # nominal dense ratio (4.5 POPS int8 / 2.25 PFLOP/s bf16)

WORKLOADS = {
    # name: (synth workload, batch)
    "decode16": ("decode", 16),
    "decode4": ("decode", 4),
    "decode1": ("decode", 1),
    "gateup": ("gateup", 2048),
    "down": ("down", 4096),
    "large": ("large", 8192),
    "tiny": ("tiny", 16),
}
# The headline line is the largest single-GPU workload (the Qwen3-32B-like MLP layer);
# the other workloads are reported in the sweep.
DEFAULT_WORKLOAD = "large"
SWEEP = ["decode16", "decode1", "decode4", "gateup", "down"]
MIN_TIMED_LAUNCHES = 200  # kernel-level timings: at least this many launches, median of replays


# ------------------------------------------------------------------ arithmetic

def weight_bytes(m, n, r):
    return m * n // 2 + 4 * (m // 128) * n + m * r // 2 + 4 * (m // 128) * r + 2 * r * n


def act_bytes(b, m, n, bf16_x=False):
    """Activation bytes of one layer call: X in (codes and scales, or BF16 X for the
    kernel that quantizes it itself) and BF16 Y out."""
    x_in = 2 * b * m if bf16_x else b * m // 2 + 4 * b * (m // 128)
    return x_in + 2 * b * n


def int8_ops(b, m, n, r):
    return 2 * b * m * n + 2 * b * m * r


def bf16_flops(b, n, r):
    return 2 * b * r * n


def describe(name):
    import synth
    wname, b = WORKLOADS[name]
    wl = synth.WORKLOADS[wname]
    return wl, b


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(
            d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


KERNEL_SOURCES = {
    # the files a capture of each kernel depends on
    "decode": ("twq_decode_sm100.cu", "sm100_ptx.cuh", "twq_eq1.cuh"),
    "pair": ("twq_pair_sm100.cu", "sm100_ptx.cuh", "twq_hrequant.cuh", "twq_eq1.cuh"),
}


def kernel_source_hash(kind):
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, "rank_residual_w4a4_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def kernel_kind(workload):
    # prefill batches of the workloads here all run on the CTA-pair kernel
    return "decode" if describe(workload.replace("_x", ""))[1] <= 16 else "pair"


def profiled_traffic(workload):
    """DRAM bytes per launch of the layer kernel from the committed ncu summary, or None
    if the summary has no line for this workload or the kernel's sources changed since."""
    p = os.path.join(ROOT, "profiles", "fused_kernel_traffic.txt")
    if not os.path.exists(p):
        return None
    want = kernel_source_hash(kernel_kind(workload))
    with open(p) as fh:
        for line in fh:
            parts = line.split()
            if len(parts) >= 3 and parts[0] == workload and not line.startswith("#"):
                if parts[2] == want:
                    return int(parts[1])
    return None


# --------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the benchmark runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            cmd = ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                   "-lms", "100"]
            if self.uuid:
                cmd += ["-i", self.uuid]
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self):
        return time.time()

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            if self.thread is not None:
                self.thread.join(timeout=2)

    def summary(self, t0, t1):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "nvidia-smi unavailable"}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, smax, reasons, power = [], [], set(), []
        for ts, line in self.lines:
            if not (t0 - 0.15 <= ts <= t1 + 0.15):
                continue
            p = [v.strip() for v in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                smax.append(float(p[2]))
                power.append(float(p[3]))
            except ValueError:
                continue
            for nm, v in zip(names, p[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "power_w_max": max(power), "samples": len(sm)}


# ---------------------------------------------------------------- distributed

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value, world, device):
    """Max of a float over ranks (identity for one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------- GPU arm

class Problem:
    """Device-resident inputs, rotating weight copies and outputs of one workload."""

    def __init__(self, name, device, seed=0, copies=None):
        import torch
        import synth
        from rank_residual_w4a4_b200 import twq
        self.name = name
        wl, b = describe(name)
        self.b, self.m, self.n, self.r = b, wl.m, wl.n, wl.r
        self.device = device
        x = synth.make_x(wl, b=b, seed=seed)
        R, L1, L2 = synth.make_weights(wl, seed=seed)
        bf = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
        self.x_host = x
        wb = weight_bytes(self.m, self.n, self.r)
        if copies is None:
            copies = max(2, min(32, math.ceil(2 * L2_BYTES / wb)))
        self.copies = copies
        w0 = twq.pack_weights(bf(R), bf(L1), bf(L2))
        self.weights = [w0] + [twq.Weights(w0.m, w0.n, w0.r, w0.rq.clone(), w0.sr.clone(),
                                           w0.l1q.clone(), w0.sl1.clone(), w0.l2t.clone())
                               for _ in range(copies - 1)]
        xd = bf(x)
        self.x = [xd] + [xd.clone() for _ in range(copies - 1)]
        self.xq = [torch.empty((b, self.m // 2), dtype=torch.uint8, device=device)
                   for _ in range(copies)]
        # prefill: the same codes one per byte (twq_quantize_act_i8), which the layer
        # kernel reads as they lie
        self.xq8 = ([torch.empty((b, self.m), dtype=torch.int8, device=device)
                     for _ in range(copies)] if b > 16 else None)
        self.sx = [torch.empty((b, self.m // 128), dtype=torch.float32, device=device)
                   for _ in range(copies)]
        self.y = [torch.empty((b, self.n), dtype=torch.bfloat16, device=device) for _ in range(copies)]
        del R, L1, L2

    @property
    def one_launch(self):
        """Decode batches: the layer kernel quantizes X itself (twq_fused_linear_x)."""
        return 1 <= self.b <= 16 and (self.r == 0 or self.r <= 128) and self.m <= 8192

    def step(self, i):
        if self.one_launch:
            self.step_x(i)
        else:
            self.step_bytes(i)

    def step_bytes(self, i):
        """Prefill: twq_quantize_act_i8 + twq_fused_linear_i8 (the codes one per byte)."""
        from rank_residual_w4a4_b200 import twq
        c = i % self.copies
        twq.quantize_act_i8(self.x[c], self.xq8[c], self.sx[c])
        twq.fused_linear_i8(self.xq8[c], self.sx[c], self.weights[c], self.y[c])

    def step_x(self, i):
        from rank_residual_w4a4_b200 import twq
        c = i % self.copies
        twq.fused_linear_x(self.x[c], self.weights[c], self.y[c])

    def step_x_a8(self, i):
        """W4A8 (8-bit activation codes), one launch: a comparison, not the metric's step."""
        from rank_residual_w4a4_b200 import twq
        c = i % self.copies
        twq.fused_linear_x(self.x[c], self.weights[c], self.y[c], a8=True)

    def step_two_call(self, i):
        from rank_residual_w4a4_b200 import twq
        c = i % self.copies
        twq.quantize_act(self.x[c], self.xq[c], self.sx[c])
        twq.fused_linear(self.xq[c], self.sx[c], self.weights[c], self.y[c])


def capture(fn, count):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="relaxed"):
        for i in range(count):
            fn(i)
    return g


def time_graph(g, world, device):
    import torch
    barrier(world)
    torch.cuda.synchronize()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record()
    g.replay()
    e.record()
    torch.cuda.synchronize()
    barrier(world)
    return s.elapsed_time(e) / 1e3  # seconds


def launch_plan(prob):
    """Launches per graph and graph replays for a kernel-level timing: a graph of
    back-to-back launches covering the weight rotation (at least 20 launches, a
    multiple of the copies), replayed until at least MIN_TIMED_LAUNCHES launches
    have been timed (at least 5 replays)."""
    per = max(prob.copies, 20 if prob.b > 16 else MIN_TIMED_LAUNCHES)
    per = -(-per // prob.copies) * prob.copies
    return per, max(5, -(-MIN_TIMED_LAUNCHES // per))


def kernel_only_time(prob, fn):
    """Median over graph replays of the seconds per launch of `fn(i)`, the launches
    captured back-to-back in one graph (no events between launches, which would
    serialize programmatically launched kernels)."""
    import torch
    per, replays = launch_plan(prob)
    g = capture(fn, per)
    g.replay()
    torch.cuda.synchronize()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    times = []
    for _ in range(replays):
        s.record()
        g.replay()
        e.record()
        torch.cuda.synchronize()
        times.append(s.elapsed_time(e) / 1e3 / per)
    del g
    return float(np.median(times))


def measure_int8_peak(device, n=8192, reps=10):
    """Dense INT8 tensor throughput of the box, measured like the BF16 entry of the
    measured peaks: torch._int_mm (cuBLASLt, int8 x int8 -> int32) on n x n x n, best
    of `reps` CUDA-event timings, in TOPS (2 n^3 ops). A roofline denominator only;
    nothing on the layer's path uses it."""
    import torch
    a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=device)
    b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=device)
    torch._int_mm(a, b)
    torch.cuda.synchronize()
    best = float("inf")
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    for _ in range(reps):
        s.record()
        torch._int_mm(a, b)
        e.record()
        torch.cuda.synchronize()
        best = min(best, s.elapsed_time(e) / 1e3)
    del a, b
    torch.cuda.empty_cache()
    return 2.0 * n ** 3 / best / 1e12


def roofline_entry(name, t_kernel, peaks, traffic, bf16_x=False, int8_measured=None):
    wl, b = describe(name)
    hbm, bf16, bf16_sus, src = peaks
    m, n, r = wl.m, wl.n, wl.r
    if b <= 64:  # decode shapes: HBM-bound
        alg = weight_bytes(m, n, r) + act_bytes(b, m, n, bf16_x)
        ach = alg / t_kernel / 1e9
        return {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(ach / hbm, 4), "traffic": traffic,
                "peak_source": "%s copy bandwidth" % src, "algorithmic_bytes": alg}
    ops = int8_ops(b, m, n, r) + bf16_flops(b, n, r)
    ach = ops / t_kernel / 1e12
    peak = bf16 * INT8_PER_BF16
    out = {"bound": "tensor", "achieved": round(ach, 1), "peak": round(peak, 1),
           "unit": "TFLOP/s", "frac": round(ach / peak, 4), "traffic": traffic,
           "peak_source": "%s bf16 burst x %g (nominal int8/bf16 dense ratio)" % (src, INT8_PER_BF16),
           "algorithmic_ops": ops}
    if int8_measured:
        out["int8_peak_measured"] = round(int8_measured, 1)
        out["frac_of_int8_measured"] = round(ach / int8_measured, 4)
    return out


def sample_rows(b, per_block=1, block=128, seed=0):
    """Rows for the output check: `per_block` seeded rows from every `block`-row block
    (every row block of the persistent schedule is looked at), plus the last row."""
    rng = np.random.default_rng(seed)
    rows = []
    for r0 in range(0, b, block):
        hi = min(b, r0 + block)
        rows.extend(sorted(rng.choice(np.arange(r0, hi), size=min(per_block, hi - r0), replace=False)))
    rows.append(b - 1)
    return np.unique(np.array(rows, dtype=np.int64))


def run_gpu(args):
    import torch
    world, rank, local = dist_setup()
    if args.gpus != world:
        raise SystemExit("bench.py: --gpus %d but %d rank(s) were launched; for N > 1 launch N "
                         "ranks with python -m torch.distributed.run --nproc-per-node N "
                         "(one process per GPU)" % (args.gpus, world))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    from rank_residual_w4a4_b200 import _build, twq
    _build.build()
    twq.load()
    peaks = load_peaks()
    int8_peak = measure_int8_peak(device)
    name = args.workload
    prob = Problem(name, device)
    K, W = args.steps, args.warmup
    wl, b = describe(name)

    # warm-up (eager once, then the warm-up graph), clock sampling from here on
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid)
    clocks.start()
    prob.step(0)
    torch.cuda.synchronize()
    gw = capture(prob.step, W)
    gk = capture(prob.step, K)
    t_load0 = time.time()
    # keep the GPU busy for a while so the clock samples see it under load
    t_end = time.time() + args.clock_seconds
    gw.replay()
    torch.cuda.synchronize()
    while time.time() < t_end:
        gw.replay()
        torch.cuda.synchronize()
    elapsed = time_graph(gk, world, device)
    t_load1 = time.time()
    elapsed = max_over_ranks(elapsed, world, device)
    del gk, gw
    # the layer kernel alone (and the quantizer alone): CUDA events around graphs of
    # back-to-back launches on the same stream and weight rotation
    def fused_only(i):
        c = i % prob.copies
        twq.fused_linear_i8(prob.xq8[c], prob.sx[c], prob.weights[c], prob.y[c])

    def quant_only(i):
        c = i % prob.copies
        twq.quantize_act_i8(prob.x[c], prob.xq8[c], prob.sx[c])

    one = prob.one_launch
    t_fused = kernel_only_time(prob, prob.step_x if one else fused_only)
    t_quant = None if one else kernel_only_time(prob, quant_only)
    # the two-call step on packed codes (twq_quantize_act + twq_fused_linear), for
    # decode and prefill batches alike
    t_two = time_graph(capture(prob.step_two_call, K), world, device) / K
    t_a8 = time_graph(capture(prob.step_x_a8, K), world, device) / K if one else None
    st = twq.device_status()
    if st != 0:
        raise RuntimeError("device wait timed out at site %d" % st)

    # the benched step once more, outside any graph, for the output check below
    prob.step(0)
    torch.cuda.synchronize()
    rows = sample_rows(b)
    y_rows = prob.y[0][torch.as_tensor(rows, device=device)].view(torch.int16).cpu().numpy().view(np.uint16)
    yf = y_rows.astype(np.uint32) << 16
    if not np.isfinite(yf.view(np.float32)).all():
        raise RuntimeError("non-finite output in the benched step: no number is reported")

    # end to end through the public C ABI, host buffers, copies inside the timed region
    e2e = run_e2e(prob, K, W, world, device)
    clocks.stop()
    clk = clocks.summary(t_load0, t_load1)

    tokens = b * world * K
    value = tokens / elapsed
    ops = int8_ops(b, wl.m, wl.n, wl.r) + bf16_flops(b, wl.n, wl.r)
    per, replays = launch_plan(prob)
    line = {
        "metric": "fused W4A4+low-rank linear: effective TOPS & tokens/s; % of HBM / INT8 roofline",
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": round(elapsed / K * 1e3, 6),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8",
        "dtype_detail": "int4 codes -> int8 MMA (s32 acc) + fp32 scales; bf16 stage 2 and output",
        "data": "synthetic (seeded generator; no dataset or trained weights)",
        "config": {"workload": "%s: b=%d m=%d n=%d r=%d, group 128" % (name, b, wl.m, wl.n, wl.r),
                   "b": b, "m": wl.m, "n": wl.n, "r": wl.r, "parallelism": "replicas x%d" % world,
                   "step": ("twq_fused_linear_x (activation quantizer inside the layer kernel)"
                            if one else "twq_quantize_act_i8 + twq_fused_linear_i8 (the 4-bit "
                            "activation codes stored one per byte; bitwise the Y of "
                            "twq_quantize_act + twq_fused_linear)"),
                   "l2": "inputs larger than L2: weights rotate over %d copies (%.0f MB > 2x L2); "
                         "X %.0f MB and Y %.0f MB per step" % (
                             prob.copies, prob.copies * weight_bytes(wl.m, wl.n, wl.r) / 1e6,
                             2 * b * wl.m / 1e6, 2 * b * wl.n / 1e6),
                   "launch": "CUDA graph of the K timed steps" + (
                       "; the layer kernel is launched with programmatic stream serialization"
                       if one else "")},
        "effective_tops": round(ops * world * K / elapsed / 1e12, 3),
        "fused_kernel_us": round(t_fused * 1e6, 3),
        "fused_kernel_timing": "median over %d replays of a graph of %d back-to-back layer "
                               "launches (%d launches timed)" % (replays, per, per * replays),
        "roofline": roofline_entry(name, t_fused, peaks,
                                   profiled_traffic(name + ("_x" if one else "")), bf16_x=one,
                                   int8_measured=int8_peak),
        "int8_peak_tops": round(int8_peak, 1),
        "int8_peak_how": "torch._int_mm 8192^3 (cuBLASLt), best of 10, CUDA events, this run",
        "e2e": e2e,
        "gpu_launches": (1 if one else 2) * K,
        "clocks": clk,
    }
    if t_quant is not None:
        line["quantize_us"] = round(t_quant * 1e6, 3)
        qb = b * wl.m * 2 + b * wl.m // 2 + 4 * b * (wl.m // 128)
        line["quantize_roofline"] = {"bound": "hbm", "achieved": round(qb / t_quant / 1e9, 1),
                                     "peak": peaks[0], "unit": "GB/s",
                                     "frac": round(qb / t_quant / 1e9 / peaks[0], 4),
                                     "algorithmic_bytes": qb}
    line["two_call_step_us"] = round(t_two * 1e6, 3)
    line["two_call_step"] = ("twq_quantize_act + twq_fused_linear (packed 4-bit activation "
                             "codes), same graph timing")
    if one:
        line["w4a8_step_us"] = round(t_a8 * 1e6, 3)
        line["w4a8_step"] = ("twq_fused_linear_x_a8: the same layer with 8-bit activation codes "
                             "(W4A8), same graph timing")
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(name, seconds=args.cpu_seconds, check=(rows, y_rows))
        line["cpu_baseline"] = cpu
        if not cpu["output_check"]["ok"]:
            raise RuntimeError("the benched step's output differs from the oracle on sampled rows "
                               "(%s): no number is reported" % json.dumps(cpu["output_check"]))
    if rank == 0 and world == 1 and not args.no_sweep:
        line["sweep"] = sweep(args, device, peaks, int8_peak)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_e2e(prob, K, W, world, device):
    """Same metric through the C ABI with host buffers: per step the H2D copy of X from
    pinned memory, the layer and the D2H copy of Y are enqueued by C-ABI calls that take
    host pointers (twq_fused_linear_x_host for decode batches, twq_linear_host otherwise),
    rotating over four streams with their own device buffers so that one stream's copies
    overlap another's kernels. Prefill batches are issued in row chunks, one call each."""
    import torch
    from rank_residual_w4a4_b200 import twq
    xh = torch.from_numpy(prob.x_host.view(np.int16)).view(torch.bfloat16).pin_memory()
    nstreams = 4
    streams = [torch.cuda.Stream(device) for _ in range(nstreams)]
    if prob.one_launch:
        xds = [torch.empty_like(prob.x[0]) for _ in streams]
        yds = [torch.empty_like(prob.y[0]) for _ in streams]
        yhs = [torch.empty((prob.b, prob.n), dtype=torch.bfloat16).pin_memory() for _ in streams]
        calls = [twq.DecodeStep(xds[j], yds[j], yhs[j], stream=streams[j]) for j in range(nstreams)]
        chunks = [(0, prob.b)]
        path = ("twq_fused_linear_x_host (H2D, the one-launch layer, D2H in one C-ABI call) via "
                "twq.DecodeStep, eager, four streams in rotation")
    else:
        chunk = max(1, min(prob.b, 1024))
        chunks = [(r0, min(prob.b, r0 + chunk)) for r0 in range(0, prob.b, chunk)]
        yh = torch.empty((prob.b, prob.n), dtype=torch.bfloat16).pin_memory()
        # chunk k always runs on stream k % 4, with its own device buffers and its own
        # rows of the pinned host Y
        calls = [twq.LinearHostStep(r1 - r0, prob.m, prob.n, device,
                                    stream=streams[k % nstreams], y_host=yh[r0:r1])
                 for k, (r0, r1) in enumerate(chunks)]
        path = ("twq_linear_host (H2D, the quantizer to codes one per byte, the layer on them, D2H, "
                "in one C-ABI call) "
                "per %d-row chunk via twq.LinearHostStep, eager, four streams in rotation" % chunk)
    xparts = [xh[r0:r1] for r0, r1 in chunks]

    def one(i):
        c = i % prob.copies
        if prob.one_launch:
            calls[i % nstreams](xparts[0], prob.weights[c])
        else:
            for k, xp in enumerate(xparts):
                calls[k](xp, prob.weights[c])

    for i in range(W):
        one(i)
    torch.cuda.synchronize()
    barrier(world)
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream()
    s.record(cur)
    for st in streams:  # the steps' streams start after s ...
        st.wait_event(s)
    h0 = time.perf_counter()
    for i in range(K):
        one(i)
    host_s = time.perf_counter() - h0  # host time to issue the K steps
    for st in streams:  # ... and e waits for all of them
        cur.wait_stream(st)
    e.record(cur)
    torch.cuda.synchronize()
    barrier(world)
    t = max_over_ranks(s.elapsed_time(e) / 1e3, world, device)
    return {"value": round(prob.b * world * K / t, 1), "unit": "tokens/s",
            "h2d_bytes_per_step": prob.b * prob.m * 2, "d2h_bytes_per_step": prob.b * prob.n * 2,
            "host_issue_us_per_step": round(host_s / K * 1e6, 2),
            "c_abi_calls_per_step": len(xparts), "path": path}


def sweep(args, device, peaks, int8_peak=None):
    """Kernel-level numbers of the other workloads: fused, w4a4_only and unfused."""
    import torch
    from rank_residual_w4a4_b200 import twq
    out = []
    names = [n for n in (args.sweep.split(",") if args.sweep else SWEEP) if n != args.workload]
    for name in names:
        prob = Problem(name, device)
        wl, b = describe(name)
        ws = torch.empty(twq.unfused_workspace_bytes(b, wl.n, wl.r), dtype=torch.uint8, device=device)
        res = {"workload": name, "b": b, "m": wl.m, "n": wl.n, "r": wl.r}

        prefill = b > 16

        def fused_packed(i):
            c = i % prob.copies
            twq.fused_linear(prob.xq[c], prob.sx[c], prob.weights[c], prob.y[c])

        def w4_packed(i):
            c = i % prob.copies
            twq.w4a4_only(prob.xq[c], prob.sx[c], prob.weights[c], prob.y[c])

        # prefill: the layer on the codes stored one per byte, and the same kernel without
        # the low-rank part (a view of the weights with r = 0), for the low-rank overhead
        w_r0 = [twq.Weights(wc.m, wc.n, 0, wc.rq, wc.sr, wc.l1q[:0], wc.sl1[:, :0], wc.l2t[:, :0])
                for wc in prob.weights]

        def fused_b(i):
            c = i % prob.copies
            twq.fused_linear_i8(prob.xq8[c], prob.sx[c], prob.weights[c], prob.y[c])

        def w4_b(i):
            c = i % prob.copies
            twq.fused_linear_i8(prob.xq8[c], prob.sx[c], w_r0[c], prob.y[c])

        def quant_b(i):
            c = i % prob.copies
            twq.quantize_act_i8(prob.x[c], prob.xq8[c], prob.sx[c])

        fused = fused_b if prefill else fused_packed
        w4 = w4_b if prefill else w4_packed

        def unf(i):
            c = i % prob.copies
            twq.unfused_linear(prob.xq[c], prob.sx[c], prob.weights[c], prob.y[c], ws)

        def quant(i):
            c = i % prob.copies
            twq.quantize_act(prob.x[c], prob.xq[c], prob.sx[c])

        # W4A8: 8-bit activation codes for the same inputs (one buffer pair per copy)
        xq8 = [torch.empty((b, wl.m), dtype=torch.int8, device=device) for _ in range(prob.copies)]
        sx8 = [torch.empty_like(prob.sx[0]) for _ in range(prob.copies)]

        def quant8(i):
            c = i % prob.copies
            twq.quantize_act_a8(prob.x[c], xq8[c], sx8[c])

        def fused8(i):
            c = i % prob.copies
            twq.fused_linear_a8(xq8[c], sx8[c], prob.weights[c], prob.y[c])

        # the INT4 stage 2 (r = 128 or 256): 4-bit L2 codes per weight copy
        s2q = wl.r in (128, 256)
        l2qs = [twq.pack_l2_int4(wc.l2t.t().contiguous()) for wc in prob.weights] if s2q else []

        def fused_s2q(i):
            c = i % prob.copies
            twq.fused_linear_s2q(prob.xq[c], prob.sx[c], prob.weights[c], l2qs[c][0], l2qs[c][1],
                                 prob.y[c])

        for i in range(prob.copies):
            quant(i)
            quant8(i)
            if prefill:
                quant_b(i)
        torch.cuda.synchronize()
        t_f = kernel_only_time(prob, fused)
        t_w = kernel_only_time(prob, w4)
        t_u = kernel_only_time(prob, unf)
        t_q = kernel_only_time(prob, quant_b if prefill else quant)
        t_fp = kernel_only_time(prob, fused_packed) if prefill else t_f
        t_x = kernel_only_time(prob, prob.step_x) if prob.one_launch else None
        t_a8 = kernel_only_time(prob, prob.step_x_a8) if prob.one_launch else None
        t_f8 = kernel_only_time(prob, fused8)
        t_s2q = kernel_only_time(prob, fused_s2q) if s2q else None
        ops = int8_ops(b, wl.m, wl.n, wl.r) + bf16_flops(b, wl.n, wl.r)
        res.update({
            "fused_us": round(t_f * 1e6, 2), "w4a4_only_us": round(t_w * 1e6, 2),
            "unfused_us": round(t_u * 1e6, 2), "quantize_us": round(t_q * 1e6, 2),
            "fused_tops": round(ops / t_f / 1e12, 2), "tokens_per_s": round(b / (t_f + t_q), 1),
            "lowrank_overhead": round(t_f / t_w - 1.0, 4), "fusion_speedup": round(t_u / t_fp, 3),
            "fused_packed_us": round(t_fp * 1e6, 2),
            "fused_input": ("the 4-bit codes one per byte (twq_fused_linear_i8); w4a4_only_us: "
                            "the same kernel with r = 0; fused_packed_us: twq_fused_linear on "
                            "packed codes; fusion_speedup: unfused over fused_packed (same input)"
                            if prefill else "packed codes (twq_fused_linear)"),
            "roofline": roofline_entry(name, t_f, peaks, profiled_traffic(name),
                                       int8_measured=int8_peak),
            "timing": "median over %d replays of a graph of %d back-to-back launches, weights "
                      "rotating over %d copies" % (launch_plan(prob)[1], launch_plan(prob)[0],
                                                  prob.copies),
            "w4a8_fused_us": round(t_f8 * 1e6, 2),
            "w4a8_roofline": roofline_entry(name, t_f8, peaks, None),
        })
        if t_s2q is not None:
            res["s2q_fused_us"] = round(t_s2q * 1e6, 2)
        if t_x is not None:
            res["fused_x_us"] = round(t_x * 1e6, 2)
            res["fused_x_a8_us"] = round(t_a8 * 1e6, 2)
            res["tokens_per_s"] = round(b / t_x, 1)
            res["roofline_x"] = roofline_entry(name, t_x, peaks, profiled_traffic(name + "_x"),
                                               bf16_x=True)
        out.append(res)
        del prob, ws, xq8, sx8, l2qs, w_r0
        torch.cuda.empty_cache()
    out.append(fold_entry(device))
    st = twq.device_status()
    if st != 0:
        raise RuntimeError("device wait timed out at site %d" % st)
    return out


# fp32 CUDA-core peak of the fold's GEMMs: 148 SMs x 128 FMA lanes x 2 flops x 1.965 GHz
FP32_ALU_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def fold_entry(device, m=4096, n=4096, r=128, reps=3):
    """The offline transform fold (U' = Q^T U G, V' = G^-1 V, R' = Q^T R) at the
    decode layer's dimensions: plain fp32 CUDA-core GEMMs, bound by fp32 issue."""
    import torch
    from rank_residual_w4a4_b200 import twq
    g = torch.Generator(device="cpu").manual_seed(0)
    Q = torch.linalg.qr(torch.randn(m, m, generator=g, dtype=torch.float64))[0].float().contiguous().to(device)
    G = (torch.eye(r, dtype=torch.float64) + 0.25 * torch.randn(r, r, generator=g, dtype=torch.float64)
         / r ** 0.5).float().to(device)
    U = (0.05 * torch.randn(m, r, generator=g)).to(torch.bfloat16).to(device)
    V = (0.05 * torch.randn(r, n, generator=g)).to(torch.bfloat16).to(device)
    R = (0.02 * torch.randn(m, n, generator=g)).to(torch.bfloat16).to(device)
    ws = torch.empty(twq.fold_workspace_bytes(m, n, r), dtype=torch.uint8, device=device)
    twq.fold_transforms(Q, G, U, V, R, ws)
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(reps):
        twq.fold_transforms(Q, G, U, V, R, ws)
    e.record()
    torch.cuda.synchronize()
    t = s.elapsed_time(e) / 1e3 / reps
    flops = 2.0 * (m * r * r + m * m * r + r * r * n + m * m * n)
    ach = flops / t / 1e12
    return {"workload": "fold m=%d n=%d r=%d" % (m, n, r), "fold_ms": round(t * 1e3, 3),
            "roofline": {"bound": "alu", "achieved": round(ach, 2), "peak": round(FP32_ALU_PEAK_TFLOPS, 1),
                         "unit": "TFLOP/s", "frac": round(ach / FP32_ALU_PEAK_TFLOPS, 4),
                         "traffic": None,
                         "peak_source": "derived: 148 SMs x 128 fp32 FMA lanes x 2 x 1.965 GHz"},
            "timing": "events around %d calls (each synchronizes once)" % reps}


# ------------------------------------------------------------- CPU oracle arm

class OracleProblem:
    """The oracle on host cores: quantize a sample of rows of X and run the layer for them."""

    def __init__(self, name, seed=0):
        import oracle
        import synth
        wl, b = describe(name)
        self.b, self.m, self.n, self.r = b, wl.m, wl.n, wl.r
        self.x = synth.make_x(wl, b=b, seed=seed)
        R, L1, L2 = synth.make_weights(wl, seed=seed)
        self.qr, self.sr = oracle.quantize_cols(R)
        self.ql1, self.sl1 = oracle.quantize_cols(L1)
        self.L2 = L2

    def rows(self, rows):
        """Y (BF16 bits) of the given rows, from BF16 X through the oracle's quantizer."""
        import oracle
        xr = self.x[rows]
        qx, sx = oracle.quantize_rows(xr)
        return oracle.linear(qx, sx, self.qr, self.sr, self.ql1, self.sl1, self.L2,
                             mode=oracle.FUSED)["y"]


def oracle_rows_parallel(op, row_lists):
    threads = [threading.Thread(target=op.rows, args=(rl,)) for rl in row_lists]
    for t in threads:
        t.start()
    for t in threads:
        t.join()


def cpu_model():
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def compare_rows(y_dev_bits, y_ref_bits):
    """The tests' Y tolerance: relative Frobenius error <= 2e-3 and per element
    |dY| <= 1e-2 rms(Y_ref) + 1 BF16 ulp of Y_ref (both against the oracle's BF16 Y)."""
    f = lambda b: (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    yd, yr = f(y_dev_bits), f(y_ref_bits)
    rms = float(np.sqrt(np.mean(yr ** 2)))
    frob = float(np.linalg.norm(yd - yr) / max(np.linalg.norm(yr), 1e-300))
    a = np.maximum(np.abs(yr), 2.0 ** -126)
    ulp = 2.0 ** (np.floor(np.log2(a)) - 7)
    excess = float((np.abs(yd - yr) - (1e-2 * rms + ulp)).max())
    ok = bool(np.isfinite(yd).all() and frob <= 2e-3 and excess <= 0.0)
    return {"ok": ok, "rows": int(y_dev_bits.shape[0]), "rel_frobenius": frob,
            "max_excess_over_elem_bound": excess}


def cpu_baseline(name, seconds=10.0, check=None):
    """The oracle timed on the host cores: a single-core leg and an all-cores leg (rows
    split over os.cpu_count() threads, each running the unmodified single-threaded
    oracle on its own rows), each about `seconds` long. With `check` = (rows, GPU Y
    bits of those rows), the oracle's Y of the same rows is compared with the GPU's."""
    op = OracleProblem(name)
    cores = os.cpu_count() or 1
    out = {"unit": "tokens/s", "cores": cores, "kind": "oracle", "cpu_model": cpu_model()}
    if check is not None:
        rows, y_dev = check
        parts = np.array_split(np.arange(rows.size), min(cores, rows.size))
        res = [None] * len(parts)

        def work(k):
            res[k] = op.rows(rows[parts[k]])

        threads = [threading.Thread(target=work, args=(k,)) for k in range(len(parts))]
        for t in threads:
            t.start()
        for t in threads:
            t.join()
        out["output_check"] = compare_rows(y_dev, np.concatenate(res, axis=0))
    # single core: calibrate on one row, then about `seconds` of rows
    t0 = time.time()
    op.rows(np.array([0]))
    per_row = max(time.time() - t0, 1e-6)
    n1 = max(1, int(seconds / per_row))
    t0 = time.time()
    op.rows(np.arange(n1) % op.b)
    t1 = time.time() - t0
    out["single_core"] = {"value": round(n1 / t1, 3), "unit": "tokens/s", "cores": 1,
                          "rows": n1}
    # all cores
    rows_per_thread = max(1, int(seconds / per_row))
    lists = [np.arange(i * rows_per_thread, (i + 1) * rows_per_thread) % op.b for i in range(cores)]
    t0 = time.time()
    oracle_rows_parallel(op, lists)
    t = time.time() - t0
    nrows = rows_per_thread * cores
    out["value"] = round(nrows / t, 3)
    out["sample"] = ("all-cores leg: %d rows of the %s workload (cycled over its %d tokens), %d "
                     "threads each running the single-threaded oracle on its own rows; single-core "
                     "leg: %d rows on one thread; weights quantized outside the timing" % (
                         nrows, name, op.b, cores, n1))
    return out


def run_reference(args):
    world, rank, _ = dist_setup()
    if rank != 0:
        return
    name = args.workload
    op = OracleProblem(name)
    cores = os.cpu_count() or 1
    rows_per_step = max(cores, min(op.b, 16))
    rows_per_step = (rows_per_step // cores) * cores
    lists_for = lambda i: [np.arange(rows_per_step // cores) + (i * rows_per_step + c * (rows_per_step // cores))
                           for c in range(cores)]
    for i in range(args.warmup):
        oracle_rows_parallel(op, [l % op.b for l in lists_for(i)])
    t0 = time.time()
    for i in range(args.steps):
        oracle_rows_parallel(op, [l % op.b for l in lists_for(i)])
    t = time.time() - t0
    wl, b = describe(name)
    value = rows_per_step * args.steps / t
    line = {
        "metric": "fused W4A4+low-rank linear: effective TOPS & tokens/s; % of HBM / INT8 roofline",
        "value": round(value, 3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(t / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64",
        "dtype_detail": "int8 codes, int64 group dot products, fp64 sums (CPU oracle)",
        "data": "synthetic (seeded generator; no dataset or trained weights)",
        "config": {"workload": "%s: b=%d m=%d n=%d r=%d, group 128" % (name, b, wl.m, wl.n, wl.r),
                   "b": b, "m": wl.m, "n": wl.n, "r": wl.r, "parallelism": "host threads"},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores,
                         "kind": "oracle", "cpu_model": cpu_model(),
                         "sample": "each step: %d rows of the %s workload over %d threads" % (
                             rows_per_step, name, cores)},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_profile(args):
    """A plain run for profilers: one copy of the workload's inputs, W + K eager calls
    of one entry point, no timing. The command lines under profiles/ use it."""
    import torch
    from rank_residual_w4a4_b200 import _build, twq
    _build.build()
    twq.load()
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    kind = args.profile
    if kind == "fold":  # the offline transform fold at the decode layer's dimensions
        res = fold_entry(device, reps=max(1, args.steps))
        print(json.dumps({"profile": kind, "fold_ms": res["fold_ms"],
                          "device_status": twq.device_status()}), flush=True)
        return
    prob = Problem(args.workload, device, copies=1)
    b, m = prob.b, prob.m
    w, x, xq, sx, y = prob.weights[0], prob.x[0], prob.xq[0], prob.sx[0], prob.y[0]
    twq.quantize_act(x, xq, sx)
    xq8 = prob.xq8[0] if prob.xq8 is not None else None
    if xq8 is not None:
        twq.quantize_act_i8(x, xq8, sx)
    extra = {}
    if kind == "a8":
        extra["xq8"], extra["sx8"] = twq.quantize_act_a8(x)
    if kind == "s2q":
        extra["l2q"], extra["sl2q"] = twq.pack_l2_int4(w.l2t.t().contiguous())
    if kind == "unfused":
        extra["ws"] = torch.empty(twq.unfused_workspace_bytes(b, prob.n, prob.r), dtype=torch.uint8,
                                  device=device)
    torch.cuda.synchronize()
    calls = {
        "step": lambda: prob.step(0),
        "quant": lambda: twq.quantize_act(x, xq, sx),
        "quant_i8": lambda: twq.quantize_act_i8(x, xq8, sx),
        "fused": lambda: twq.fused_linear(xq, sx, w, y),
        "fused_i8": lambda: twq.fused_linear_i8(xq8, sx, w, y),
        "w4a4": lambda: twq.w4a4_only(xq, sx, w, y),
        "lowrank": lambda: twq.lowrank_only(xq, sx, w, y),
        "fused_x": lambda: twq.fused_linear_x(x, w, y),
        "a8": lambda: twq.fused_linear_a8(extra["xq8"], extra["sx8"], w, y),
        "s2q": lambda: twq.fused_linear_s2q(xq, sx, w, extra["l2q"], extra["sl2q"], y),
        "unfused": lambda: twq.unfused_linear(xq, sx, w, y, extra["ws"]),
    }
    for _ in range(args.warmup + args.steps):
        calls[kind]()
    torch.cuda.synchronize()
    st = twq.device_status()
    print(json.dumps({"profile": kind, "workload": args.workload, "calls": args.warmup + args.steps,
                      "device_status": st}), flush=True)
    if st != 0:
        raise SystemExit(1)


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["twq", "reference"], default="twq")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--sweep", default="", help="comma-separated workloads for the sweep")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--clock-seconds", type=float, default=1.0,
                    help="seconds of warm-up replays before the timed region (clock sampling)")
    ap.add_argument("--profile", choices=["step", "quant", "quant_i8", "fused", "fused_i8", "w4a4",
                                          "lowrank", "fused_x", "a8", "s2q", "unfused", "fold"],
                    help="plain run for a profiler: W + K eager calls of one entry point on one "
                         "copy of the inputs, no timing")
    args = ap.parse_args()
    if args.profile:
        run_profile(args)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
