"""Benchmark of the LLM.int8() mixed-precision linear on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {ours,reference}]

One step = the four BLOOM-176B block linears (QKV 43008x14336, attn-out
14336x14336, fc1 57344x14336, fc2 14336x57344) at 2048 tokens, each a full
llmint8_matmul_mixed call: fused quantizer + outlier detection, fix-up and
compaction, and the tcgen05 int8 GEMM with the fused dequant + fp16 outlier
epilogue. Inputs are seeded synthetic data with the workload's outlier columns
(~0.05% of hidden columns x60), threshold 6.0, weights random N(0, 0.02)
quantized once per output row before timing (offline weight preparation).

Metric: int8-mixed linear TOPS = sum of 2*M*N*K over the four linears per
step / step time. Every linear's int8 weight (205-822 MB) is larger than L2,
so no explicit flush is needed between iterations.

--impl reference times the CPU oracle (plain single-threaded C, the
definition the GPU path is checked against) on a bounded sample of the same
workload: all 2048 tokens against a slice of each weight's output rows.

Multi-GPU: the layer has no exchange step on this path; `--gpus N` (under
torchrun) runs one independent replica per GPU and reports the aggregate.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

WORKLOAD = synthetic.BLOOM_BLOCK_2048
METRIC = "int8-mixed linear TOPS (BLOOM-176B block linears, 2048 tokens)"
UNIT = "TOPS"
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "k_gemm_i8_bloom_block_traffic.txt")
GEMM_SOURCES = [os.path.join(ROOT, "int8_mixed_precision_rowwise_b200", "csrc", f)
                for f in ("gemm.cu", "ptx.cuh", "sched.h")]
CLOCK_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def ops_of(lin) -> int:
    return 2 * lin.M * lin.N * lin.K


def workload_config(extra=None):
    cfg = {
        "workload": WORKLOAD.name,
        "linears": {l.name: [l.M, l.N, l.K] for l in WORKLOAD.linears},
        "tokens": WORKLOAD.linears[0].M,
        "threshold": WORKLOAD.threshold,
        "outlier_cols": {l.name: l.n_outlier_cols for l in WORKLOAD.linears},
        "outlier_scale": 60.0,
        "weights": "fp16 N(0,0.02) kept for outlier columns; int8 CB/SCB prepared before timing",
        "l2": "no flush: each linear's int8 weight (205-822 MB) exceeds the 126 MB L2",
    }
    if extra:
        cfg.update(extra)
    return cfg


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def gemm_source_hash() -> str:
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per GEMM launch from the committed ncu summary, or None if
    the summary is missing or the kernel source changed since the capture."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    vals = {}
    with open(TRAFFIC_FILE) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("gemm_source_sha256_16") != gemm_source_hash():
        return None
    try:
        return float(vals["dram_bytes_per_launch_avg"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi samples every 50 ms while the timed region runs."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={CLOCK_QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            # the region starts once nvidia-smi delivers samples (it takes a
            # moment to start), so that short regions are covered too
            t0 = time.time()
            while not self.lines and time.time() - t0 < 3.0 and self.proc.poll() is None:
                time.sleep(0.01)
            self.skip = len(self.lines)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines[getattr(self, "skip", 0):]:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            why = ("no clock sample during the timed region (shorter than nvidia-smi's first sample)"
                   if self.proc is not None else "nvidia-smi unavailable")
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [why], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- GPU arm

def max_over_ranks(values, world, device):
    """Each timing's maximum over the ranks (the slowest replica sets the
    job's time); unchanged with one rank."""
    import torch
    import torch.distributed as dist

    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_tops(world, ops_per_step, steps, ms_total):
    """Whole-job throughput: every replica's work over the slowest replica's time."""
    return world * ops_per_step * steps / (ms_total * 1e-3) / 1e12


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import int8_mixed_precision_rowwise_b200 as L

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peaks, peak_kind = load_peaks()
    int8_peak_burst = 2.0 * peaks["bf16_tflops"]          # nominal int8 : bf16 = 4.5 : 2.25
    int8_peak_sustained = 2.0 * peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])

    # Inputs resident in HBM; weights prepared (quantized per output row) once.
    layers, xs, ys = [], [], []
    for li, lin in enumerate(WORKLOAD.linears):
        X, W, _ = synthetic.torch_device_problem(lin, seed=100 + li + 17 * rank, device=dev)
        layers.append(L.Int8MixedLinear.from_fp16(W, WORKLOAD.threshold, keep_fp16_weights=True))
        xs.append(X)
        ys.append(torch.empty((lin.M, lin.N), dtype=torch.float16, device=dev))
    torch.cuda.synchronize()
    step_ops = sum(ops_of(l) for l in WORKLOAD.linears)
    nlin = len(WORKLOAD.linears)
    ev_b = [[torch.cuda.Event(enable_timing=True) for _ in range(nlin)] for _ in range(args.steps)]
    ev_e = [[torch.cuda.Event(enable_timing=True) for _ in range(nlin)] for _ in range(args.steps)]
    for row in ev_b + ev_e:
        for e in row:
            e.record()

    def step(k=None):
        for i, layer in enumerate(layers):
            dbg = None if k is None else {"gemm_begin": ev_b[k][i], "gemm_end": ev_e[k][i]}
            L.matmul_mixed(xs[i], layer.CB, layer.SCB, layer.W_f16, layer.threshold, Y=ys[i], debug=dbg)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clocks:
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        t0.record()
        for k in range(args.steps):
            step(k)
        t1.record()
        torch.cuda.synchronize()
    ms_total = t0.elapsed_time(t1)
    gemm_ms = sum(ev_b[k][i].elapsed_time(ev_e[k][i]) for k in range(args.steps) for i in range(nlin))
    for ws in L.workspaces(local_rank):
        status = L.read_status(ws, clear=False)
        if status:
            raise RuntimeError(f"device status word {status:#x}: a kernel gave up on a bounded wait")

    # e2e: the same step through the public API with host buffers: X from pinned
    # host memory to the device, the layer, Y back to pinned host memory. The
    # copies run on streams of their own (PCIe is full duplex: inputs in and
    # outputs out at once) and overlap the layers: linear i's X goes in while
    # earlier linears compute, its Y comes out while later ones do. Every
    # step still moves all of its inputs in and all of its outputs out.
    xh = [x.cpu().pin_memory() for x in xs]
    yh = [torch.empty(y.shape, dtype=y.dtype, pin_memory=True) for y in ys]
    xd = [torch.empty_like(x) for x in xs]
    yd = [torch.empty_like(y) for y in ys]
    e2e_steps = max(3, min(args.steps, 20))
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    nl = len(layers)
    ev_in = [torch.cuda.Event() for _ in range(nl)]
    ev_cmp = [torch.cuda.Event() for _ in range(nl)]
    ev_out = [torch.cuda.Event() for _ in range(nl)]
    started = [False]

    def e2e_step():
        for i in range(nl):
            with torch.cuda.stream(s_in):
                if started[0]:
                    s_in.wait_event(ev_cmp[i])   # the previous step's layer i has read xd[i]
                xd[i].copy_(xh[i], non_blocking=True)
                ev_in[i].record(s_in)
        for i, layer in enumerate(layers):
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev_in[i])
                if started[0]:
                    s_cmp.wait_event(ev_out[i])  # the previous step's Y of layer i is out
                layer(xd[i], yd[i])
                ev_cmp[i].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[i])
                yh[i].copy_(yd[i], non_blocking=True)
                ev_out[i].record(s_out)
        started[0] = True

    cur = torch.cuda.current_stream(dev)
    for s_ in (s_in, s_cmp, s_out):
        s_.wait_stream(cur)
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(cur)
    for s_ in (s_in, s_cmp, s_out):
        s_.wait_stream(cur)
    for _ in range(e2e_steps):
        e2e_step()
    for s_ in (s_in, s_cmp, s_out):
        cur.wait_stream(s_)
    b.record(cur)
    torch.cuda.synchronize()
    e2e_ms = a.elapsed_time(b) / e2e_steps
    # the host copies hold what the device computed
    if not all(torch.equal(yh[i], yd[i].cpu()) for i in range(nl)):
        raise RuntimeError("end-to-end outputs on the host differ from the device's")

    int8_measured = measure_int8_peak(dev, local_rank) if rank == 0 else None
    secondary = measure_secondary(L, dev, local_rank) if rank == 0 else None

    ms_total, gemm_ms, e2e_ms = max_over_ranks([ms_total, gemm_ms, e2e_ms], world, dev)
    if rank != 0:
        return None
    ms_step = ms_total / args.steps
    value = whole_job_tops(world, step_ops, args.steps, ms_total)
    gemm_launches = args.steps * nlin
    achieved = step_ops * args.steps / (gemm_ms * 1e-3) / 1e12
    traffic = recorded_traffic()
    clk = clocks.summary()
    peak, peak_choice = pick_int8_peak(int8_peak_burst, int8_peak_sustained, clk, ms_total * 1e-3,
                                       peaks.get("sm_max_mhz"))
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": workload_config({"parallelism": f"replicas{world}" if world > 1 else "single"}),
        "roofline": {
            "bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": "TOPS",
            "frac": round(achieved / peak, 4), "traffic": traffic,
            "kernel": "k_gemm_i8_pair (CTA-pair tcgen05 int8 GEMM, fused dequant + outlier epilogue)",
            "peak_source": f"2 x bf16 {peak_choice['kind']} of {peak_kind} (bf16 {peaks.get('bf16_tflops')} burst / "
                           f"{peaks.get('bf16_tflops_sustained')} sustained TF/s), nominal int8:bf16 = 4.5:2.25",
            "peak_choice": peak_choice["why"],
            "peak_burst": round(int8_peak_burst, 1), "peak_sustained": round(int8_peak_sustained, 1),
            "frac_of_spec_4500": round(achieved / 4500.0, 4),
            "int8_measured": int8_measured,
            "frac_of_int8_measured": (round(achieved / int8_measured["tops"], 4)
                                      if int8_measured and int8_measured.get("tops") else None),
        },
        "gemm_share_of_step": round(gemm_ms / ms_total, 4),
        "cpu_baseline": cpu_baseline(args) if world == 1 else None,
        "e2e": {"value": round(world * step_ops / (e2e_ms * 1e-3) / 1e12, 3), "unit": UNIT,
                "h2d_bytes_per_step": int(sum(x.numel() * 2 for x in xs)),
                "d2h_bytes_per_step": int(sum(y.numel() * 2 for y in ys))},
        # per linear: the streaming quantizer, the outlier-operand gather and the GEMM
        # (the bitmap clear before the quantizer is a cudaMemsetAsync, not a kernel of ours)
        "gpu_launches": 3 * gemm_launches,
        "clocks": {"sm_mhz": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"], "reasons": clk["reasons"]},
        "secondary": secondary,
    }
    return line


def pick_int8_peak(burst, sustained, clk, timed_s, sm_max):
    """The int8 denominator that matches the clocks the timed region ran at:
    the burst figure when the median SM clock sat at (within 5% of) its
    maximum, the sustained one when it sat below (the power cap pulled it
    down), and, with no clock sample, burst for a region under a second (too
    short for the cap to act) and sustained otherwise."""
    sm = clk.get("sm_mhz")
    mx = clk.get("sm_max_mhz") or sm_max
    if sm is not None and mx:
        if sm >= 0.95 * mx:
            return burst, {"kind": "burst", "why": f"median SM clock {sm:.0f} MHz at its maximum {mx:.0f} MHz"}
        return sustained, {"kind": "sustained",
                           "why": f"median SM clock {sm:.0f} MHz below its maximum {mx:.0f} MHz (power cap)"}
    if timed_s < 1.0:
        return burst, {"kind": "burst", "why": f"no clock sample; timed region {timed_s:.3f} s, under 1 s"}
    return sustained, {"kind": "sustained", "why": f"no clock sample; timed region {timed_s:.1f} s"}


def measure_int8_peak(dev, index, reps=10):
    """A measured int8 tensor-core rate on this GPU: cuBLAS's int8 GEMM
    (torch._int_mm, int32 out) on the fc1 shape 2048 x 57344 x 14336, timed
    alone with CUDA events, best of `reps`, for the weight operand both
    column-major (a transposed view) and row-major; the faster layout counts."""
    import torch

    lin = {l.name: l for l in WORKLOAD.linears}["fc1"]
    M, N, K = lin.M, lin.N, lin.K
    g = torch.Generator(device=dev)
    g.manual_seed(5)
    A = torch.randint(-127, 128, (M, K), generator=g, device=dev, dtype=torch.int8)
    B = torch.randint(-127, 128, (N, K), generator=g, device=dev, dtype=torch.int8)
    out = {"routine": "torch._int_mm (cuBLAS int8, int32 out)", "shape": [M, N, K]}
    best = None
    with ClockSampler(index) as clocks:
        for layout, b in (("B column-major", B.t()), ("B row-major", B.t().contiguous())):
            try:
                for _ in range(2):
                    torch._int_mm(A, b)
                torch.cuda.synchronize()
                ts = []
                for _ in range(reps):
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record()
                    torch._int_mm(A, b)
                    e1.record()
                    torch.cuda.synchronize()
                    ts.append(e0.elapsed_time(e1))
                tops = 2 * M * N * K / (min(ts) * 1e-3) / 1e12
                out[layout] = round(tops, 1)
                if best is None or tops > best:
                    best = tops
            except RuntimeError as e:
                out[layout] = f"failed: {str(e).splitlines()[0][:120]}"
            del b
    del A, B
    torch.cuda.empty_cache()
    out["tops"] = round(best, 1) if best else None
    out["clocks"] = clocks.summary()
    return out


def per_linear_times(L, dev, reps=10):
    """For each BLOOM linear and the 2048 x 16384 x 4096 prefill linear: the
    GEMM alone (events around its launch) and the whole llmint8_matmul_mixed
    call (quantizer, GEMM), median of `reps` calls; int8 TOPS of each."""
    import torch

    res = {}
    lins = list(WORKLOAD.linears) + list(synthetic.PREFILL_7B.linears)
    for li, lin in enumerate(lins):
        X, W, _ = synthetic.torch_device_problem(lin, seed=200 + li, device=dev)
        layer = L.Int8MixedLinear.from_fp16(W, WORKLOAD.threshold, keep_fp16_weights=True)
        Y = torch.empty((lin.M, lin.N), dtype=torch.float16, device=dev)
        gb = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
        ge = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
        cb = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
        ce = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
        for _ in range(2):
            L.matmul_mixed(X, layer.CB, layer.SCB, layer.W_f16, layer.threshold, Y=Y)
        torch.cuda.synchronize()
        for k in range(reps):
            cb[k].record()
            L.matmul_mixed(X, layer.CB, layer.SCB, layer.W_f16, layer.threshold, Y=Y,
                           debug={"gemm_begin": gb[k], "gemm_end": ge[k]})
            ce[k].record()
        torch.cuda.synchronize()
        gemm_us = statistics.median(gb[k].elapsed_time(ge[k]) for k in range(reps)) * 1e3
        call_us = statistics.median(cb[k].elapsed_time(ce[k]) for k in range(reps)) * 1e3
        ops = ops_of(lin)
        name = lin.name if lin in WORKLOAD.linears else f"prefill_{lin.M}x{lin.N}x{lin.K}"
        res[name] = {"gemm_us": round(gemm_us, 1), "gemm_tops": round(ops / (gemm_us * 1e-6) / 1e12, 1),
                     "call_us": round(call_us, 1), "call_tops": round(ops / (call_us * 1e-6) / 1e12, 1)}
        del layer, X, W, Y
    torch.cuda.empty_cache()
    return res


def graph_time_ms(fns, reps, min_s=0.3):
    """Average device time per call of `fns` (called in turn, `reps` times),
    captured into one CUDA graph so host launch overhead is excluded; the
    calls rotate over inputs larger than L2 together. The graph is replayed
    for at least `min_s` seconds (so that the clock sampler sees the load);
    the median replay counts."""
    import torch

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for f in fns:  # first calls outside capture (per-device set-up)
            f()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(reps):
            for f in fns:
                f()
    g.replay()
    torch.cuda.synchronize()
    ts = []
    t_start = time.time()
    while len(ts) < 3 or (time.time() - t_start < min_s and len(ts) < 5000):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b) / (reps * len(fns)))
    del g
    return statistics.median(ts)


def measure_secondary(L, dev, index):
    """The quantizer (4096 x 4096, 8 columns x40) and the decode path (BLOOM
    width, M = 1, 8, 32) in HBM GB/s of algorithmic bytes. Each is timed as a
    CUDA graph of back-to-back calls; the quantizer rotates over 8 inputs
    (256 MB, twice L2), the decode weights (205 MB) exceed L2 by themselves.
    The 2048 x 16384 x 4096 prefill linear (TOPS) is timed the same way (its
    output, 67 MB, and weight, 67 MB, together exceed L2). Every leg carries
    the SM clocks sampled while it ran."""
    import torch

    peaks, _ = load_peaks()
    hbm = peaks["hbm_gbs"]
    out = {"timing": "CUDA graph of back-to-back calls, replayed >= 0.3 s, median replay; inputs larger than L2",
           "hbm_peak_gbs": hbm}
    lin = synthetic.QUANT_4096.linears[0]
    bufs = []
    for k in range(8):
        X, _, _ = synthetic.torch_device_problem(
            synthetic.Linear("q", lin.M, 1, lin.K, lin.n_outlier_cols, lin.outlier_scale), k, dev)
        bufs.append((X, torch.empty((lin.M, lin.K), dtype=torch.int8, device=dev),
                     torch.empty(lin.M, dtype=torch.float32, device=dev),
                     torch.empty((lin.K + 31) // 32, dtype=torch.int32, device=dev)))
    fns = [lambda b=b: L.quantize_rowwise(b[0], 6.0, b[1], b[2], b[3]) for b in bufs]
    with ClockSampler(index) as clk:
        ms = graph_time_ms(fns, reps=4)
    byts = 2 * lin.M * lin.K + lin.M * lin.K + 4 * lin.M + lin.K // 8
    out["quantizer_4096x4096"] = {"us": round(ms * 1e3, 2), "GBs": round(byts / (ms * 1e-3) / 1e9, 1),
                                  "frac": round(byts / (ms * 1e-3) / 1e9 / hbm, 3), "clocks": clk.summary()}
    del bufs, fns
    for M in (1, 8, 32):
        lin = synthetic.decode_bloom(M).linears[0]
        X, W, _ = synthetic.torch_device_problem(lin, 0, dev)
        layer = L.Int8MixedLinear.from_fp16(W, keep_fp16_weights=False)
        del W
        Y = torch.empty((M, lin.N), dtype=torch.float16, device=dev)
        with ClockSampler(index) as clk:
            ms = graph_time_ms([lambda: layer(X, Y)], reps=20)
        byts = lin.N * lin.K + 4 * lin.N + 2 * M * lin.K + 2 * M * lin.N
        out[f"decode_M{M}"] = {"us": round(ms * 1e3, 2), "GBs": round(byts / (ms * 1e-3) / 1e9, 1),
                               "frac": round(byts / (ms * 1e-3) / 1e9 / hbm, 3), "clocks": clk.summary()}
        del layer, X, Y
    torch.cuda.empty_cache()
    # The 7B-class prefill linear (2048 x 16384 x 4096) through llmint8_matmul_mixed:
    # quantizer, outlier gather and GEMM back to back, as in the zero-point leg below.
    lin = synthetic.PREFILL_7B.linears[0]
    X, W, _ = synthetic.torch_device_problem(lin, 0, dev)
    layer = L.Int8MixedLinear.from_fp16(W, 6.0, keep_fp16_weights=True)
    del W
    Y = torch.empty((lin.M, lin.N), dtype=torch.float16, device=dev)
    with ClockSampler(index) as clk:
        ms = graph_time_ms([lambda: layer(X, Y)], reps=10)
    out["prefill_2048x16384x4096"] = {"call_us": round(ms * 1e3, 1),
                                      "call_tops": round(ops_of(lin) / (ms * 1e-3) / 1e12, 1),
                                      "clocks": clk.summary()}
    del layer, X, Y
    torch.cuda.empty_cache()
    out["zero_point"] = zero_point_times(L, dev, hbm, index)
    # Last: the per-linear GEMMs run the GPU at its power cap for seconds.
    with ClockSampler(index) as clk:
        out["per_linear"] = per_linear_times(L, dev)
    out["per_linear"]["clocks"] = clk.summary()
    return out


def zero_point_times(L, dev, hbm, index):
    """The zero-point variant: its quantizer on 4096 x 4096 (GB/s of the same
    algorithmic bytes plus the zero points) and the whole linear on the
    2048 x 16384 x 4096 prefill shape (TOPS), both CUDA-graph timed."""
    import torch

    res = {}
    lin = synthetic.QUANT_4096.linears[0]
    bufs = []
    for k in range(8):
        X, _, _ = synthetic.torch_device_problem(
            synthetic.Linear("q", lin.M, 1, lin.K, lin.n_outlier_cols, lin.outlier_scale), k, dev)
        bufs.append((X, torch.empty((lin.M, lin.K), dtype=torch.int8, device=dev),
                     torch.empty(lin.M, dtype=torch.float32, device=dev),
                     torch.empty(lin.M, dtype=torch.int32, device=dev),
                     torch.empty((lin.K + 31) // 32, dtype=torch.int32, device=dev)))
    fns = [lambda b=b: L.quantize_rowwise_asym(b[0], 6.0, b[1], b[2], b[3], b[4]) for b in bufs]
    with ClockSampler(index) as clk:
        ms = graph_time_ms(fns, reps=4)
    byts = 2 * lin.M * lin.K + lin.M * lin.K + 8 * lin.M + lin.K // 8
    res["quantizer_4096x4096"] = {"us": round(ms * 1e3, 2), "GBs": round(byts / (ms * 1e-3) / 1e9, 1),
                                  "frac": round(byts / (ms * 1e-3) / 1e9 / hbm, 3), "clocks": clk.summary()}
    del bufs, fns
    lin = synthetic.Linear("prefill", 2048, 16384, 4096, 4, 60.0)
    X, W, _ = synthetic.torch_device_problem(lin, 0, dev)
    CB, SCB, _ = L.quantize_rowwise(W, 0.0)
    R = L.code_row_sums(CB)
    Y = torch.empty((lin.M, lin.N), dtype=torch.float16, device=dev)
    with ClockSampler(index) as clk:
        ms = graph_time_ms([lambda: L.matmul_mixed_asym(X, CB, SCB, R, W, 6.0, Y=Y)], reps=10)
    res["prefill_2048x16384x4096"] = {"call_us": round(ms * 1e3, 1),
                                      "call_tops": round(ops_of(lin) / (ms * 1e-3) / 1e12, 1),
                                      "clocks": clk.summary()}
    del X, W, CB, SCB, R, Y
    torch.cuda.empty_cache()
    return res


# --------------------------------------------------------------------------- CPU oracle arm

SAMPLE_COLS = 128  # weight output rows per linear in the CPU sample


def oracle_sample_step(oracle, lin, li):
    """The oracle's whole linear on all tokens against SAMPLE_COLS weight rows.
    Returns the algorithmic ops it covered."""
    X, _ = synthetic.make_activations(lin, seed=100 + li)
    W = synthetic.make_weight(lin, seed=100 + li, rows=SAMPLE_COLS)
    oracle.matmul_mixed(X, WORKLOAD.threshold, W=W)
    return 2 * lin.M * SAMPLE_COLS * lin.K


def host_info():
    """The host the oracle runs on: logical CPUs the process may use, the CPU
    model, and the threads the oracle uses (it is single-threaded C)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        usable = len(os.sched_getaffinity(0))
    except AttributeError:
        usable = os.cpu_count()
    return {"nproc": usable, "cpu_count": os.cpu_count(), "cpu_model": model, "oracle_threads": 1}


def oracle_full_configs(oracle):
    """The oracle timed on whole workloads that it finishes in seconds: the
    tiny linear (8 x 64 -> 128), the 4096 x 4096 quantizer and the decode
    linears at BLOOM width (M = 1, 8, 32 against a 14336 x 14336 int8
    weight), each in the metric the GPU lines report (us, GB/s of the same
    algorithmic bytes). Weight preparation (quantizing W) is not timed."""
    res = {}
    lin = synthetic.TINY.linears[0]
    X16, W16, _ = synthetic.make_problem(lin, seed=0)
    n, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < 0.5:
        oracle.matmul_mixed(X16, synthetic.TINY.threshold, W=W16)
        n += 1
    res["tiny_8x64x128"] = {"us": round((time.perf_counter() - t0) / n * 1e6, 1), "calls": n}
    lin = synthetic.QUANT_4096.linears[0]
    X16, _ = synthetic.make_activations(lin, seed=0)
    t0 = time.perf_counter()
    O = oracle.outlier_cols(X16, 6.0)
    oracle.quantize_rowwise(X16, O)
    sec = time.perf_counter() - t0
    byts = 2 * lin.M * lin.K + lin.M * lin.K + 4 * lin.M + lin.K // 8
    res["quantizer_4096x4096"] = {"ms": round(sec * 1e3, 1), "GBs": round(byts / sec / 1e9, 3)}
    dlin = synthetic.decode_bloom(1).linears[0]
    W16 = synthetic.make_weight(dlin, seed=0)
    CB, SB = oracle.quantize_weight(W16)
    del W16
    for M in (1, 8, 32):
        lin = synthetic.decode_bloom(M).linears[0]
        X16, _ = synthetic.make_activations(lin, seed=M)
        t0 = time.perf_counter()
        oracle.matmul_mixed(X16, 6.0, CB=CB, SB=SB)
        sec = time.perf_counter() - t0
        byts = lin.N * lin.K + 4 * lin.N + 2 * M * lin.K + 2 * M * lin.N
        res[f"decode_M{M}"] = {"ms": round(sec * 1e3, 1), "GBs": round(byts / sec / 1e9, 3)}
    return res


def cpu_baseline(args, steps=1):
    import oracle

    oracle.build()
    ops, secs = 0, 0.0
    for _ in range(steps):
        for li, lin in enumerate(WORKLOAD.linears):
            X, _ = synthetic.make_activations(lin, seed=100 + li)
            W = synthetic.make_weight(lin, seed=100 + li, rows=SAMPLE_COLS)
            t0 = time.perf_counter()
            oracle.matmul_mixed(X, WORKLOAD.threshold, W=W)
            secs += time.perf_counter() - t0
            ops += 2 * lin.M * SAMPLE_COLS * lin.K
    host = host_info()
    return {"value": round(ops / secs / 1e12, 6), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"all {WORKLOAD.linears[0].M} tokens x {SAMPLE_COLS} output rows of each of the four "
                      f"linears (full outlier detection and quantization of X), single-threaded C, "
                      f"{secs:.1f} s",
            "host": host, "full_configs": oracle_full_configs(oracle)}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    import oracle

    oracle.build()
    for _ in range(args.warmup):
        oracle_sample_step(oracle, WORKLOAD.linears[1], 1)
    ops, secs = 0, 0.0
    for _ in range(args.steps):
        for li, lin in enumerate(WORKLOAD.linears):
            X, _ = synthetic.make_activations(lin, seed=100 + li)
            W = synthetic.make_weight(lin, seed=100 + li, rows=SAMPLE_COLS)
            t0 = time.perf_counter()
            oracle.matmul_mixed(X, WORKLOAD.threshold, W=W)
            secs += time.perf_counter() - t0
            ops += 2 * lin.M * SAMPLE_COLS * lin.K
    value = ops / secs / 1e12
    sample = (f"each step: all {WORKLOAD.linears[0].M} tokens x {SAMPLE_COLS} output rows of each of the four "
              f"linears, single-threaded C oracle")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs / args.steps * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": workload_config({"parallelism": "single"}),
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample,
                         "host": host_info()},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_profile_case(args):
    """A minimal driver for ncu captures: set up the named BLOOM linear (or
    'all' four, or 'prefill' for the 2048 x 16384 x 4096 linear), run one
    warm-up pass, then --steps passes inside an NVTX range 'timed_steps'.
    Prints nothing; exits 0 on success."""
    import torch

    import int8_mixed_precision_rowwise_b200 as L

    dev = torch.device("cuda", 0)
    if args.profile_case == "quantizer":
        lin = synthetic.QUANT_4096.linears[0]
        X, _, _ = synthetic.torch_device_problem(
            synthetic.Linear("q", lin.M, 1, lin.K, lin.n_outlier_cols, lin.outlier_scale), 0, dev)
        L.quantize_rowwise(X, 6.0)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_push("timed_steps")
        for _ in range(args.steps):
            L.quantize_rowwise(X, 6.0)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
        return
    if args.profile_case.startswith("cublas_int8_"):
        # cuBLAS's int8 GEMM (torch._int_mm) on a BLOOM linear's shape: the
        # library kernel the measured int8 peak comes from, for comparison.
        lin = {l.name: l for l in WORKLOAD.linears}[args.profile_case[len("cublas_int8_"):]]
        g = torch.Generator(device=dev)
        g.manual_seed(5)
        A = torch.randint(-127, 128, (lin.M, lin.K), generator=g, device=dev, dtype=torch.int8)
        B = torch.randint(-127, 128, (lin.N, lin.K), generator=g, device=dev, dtype=torch.int8).t()
        torch._int_mm(A, B)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_push("timed_steps")
        for _ in range(args.steps):
            torch._int_mm(A, B)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
        return
    if args.profile_case.startswith("decode_M"):
        lin = synthetic.decode_bloom(int(args.profile_case[len("decode_M"):])).linears[0]
        X, W, _ = synthetic.torch_device_problem(lin, 0, dev)
        layer = L.Int8MixedLinear.from_fp16(W, keep_fp16_weights=False)
        del W
        layer(X)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_push("timed_steps")
        for _ in range(args.steps):
            layer(X)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
        return
    lins = [l for l in WORKLOAD.linears if args.profile_case in ("all", l.name)]
    if args.profile_case == "prefill":
        lins = list(synthetic.PREFILL_7B.linears)
    if not lins:
        raise SystemExit(f"unknown case {args.profile_case!r}")
    layers, xs, ys = [], [], []
    for li, lin in enumerate(lins):
        X, W, _ = synthetic.torch_device_problem(lin, seed=100 + li, device=dev)
        layers.append(L.Int8MixedLinear.from_fp16(W, WORKLOAD.threshold, keep_fp16_weights=True))
        xs.append(X)
        ys.append(torch.empty((lin.M, lin.N), dtype=torch.float16, device=dev))
    for i, layer in enumerate(layers):
        layer(xs[i], ys[i])
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("timed_steps")
    for _ in range(args.steps):
        for i, layer in enumerate(layers):
            layer(xs[i], ys[i])
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    assert all(L.read_status(ws, clear=False) == 0 for ws in L.workspaces(0))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--profile-case", default=None,
                    help="ncu driver: run only this BLOOM linear ('qkv', 'attn_out', 'fc1', 'fc2' or 'all'), "
                         "the 2048 x 16384 x 4096 'prefill' linear, the 4096 x 4096 'quantizer', "
                         "'decode_M1' / 'decode_M8' / 'decode_M32', or "
                         "cuBLAS's int8 GEMM on a linear's shape ('cublas_int8_attn_out', ...)")
    args = ap.parse_args()
    if args.profile_case:
        run_profile_case(args)
        return
    args.warmup = max(args.warmup, 3) if args.impl == "ours" else args.warmup

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and world > 1:
        print(f"warning: WORLD_SIZE={world} but --gpus {args.gpus}", file=sys.stderr)

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist
    from datetime import timedelta

    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
