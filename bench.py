"""Benchmark of the NVFP4 W4A4 linear layer on B200.

One step = the whole hot path over one batch: quantize the activation to
NVFP4 (E4M3 block scales, static calibrated global scale), block-scaled
FP4 GEMM against a pre-quantized weight, dequantizing BF16 epilogue.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode]
                    [--impl reference] [--no-extra] [--no-cpu-baseline]

The headline line is the decode-shape linear (X[8,5120] x W[12288,5120],
HBM-bound, GB/s).  Prefill (32768x17408x5120, TFLOP/s), the fused GDN
projection and the quantize sweep are measured too and reported under
"extra".  Inputs are seeded synthetic tensors already resident in HBM; the
decode weight rotates through enough copies to exceed 3x the L2 size, so
no step reads a weight left in L2 by the previous step.

Multi-GPU (torchrun): every rank runs its own replica on its own batch (the
layer has no exchange step); value = all ranks' bytes / max-over-ranks time.
``--impl reference`` times the CPU oracle (the plain C reference) on the
host on the same workload instead.
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

METRIC = "NVFP4 W4A4 GEMM TFLOPS (prefill) & GB/s (decode) vs B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP4_OVER_BF16 = 4.0          # nominal dense FP4 : BF16 tensor throughput (9 : 2.25 PFLOP/s)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


# The sources each kernel's recorded counters depend on.
KERNEL_SOURCES = {
    "nvfp4_gemm_kernel": ("gemm.cu", "block_quant.cuh", "ptx.cuh", "common.h", "runtime.cu"),
    "quantize_kernel": ("quantize.cu", "block_quant.cuh", "ptx.cuh", "common.h"),
}


def source_hash(kernel: str, read=None) -> str:
    """Hash of one kernel's sources with // comments and blank lines removed,
    so that a comment edit, or a change to another kernel, keeps its recorded
    counters valid.  read(name) -> text overrides reading the working tree."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        if read is None:
            with open(os.path.join(ROOT, "nvfp4_w4a4_quantized_10_b200", "csrc", name), encoding="utf-8") as f:
                text = f.read()
        else:
            text = read(name)
        for line in text.splitlines():
            code = line.split("//", 1)[0].rstrip()
            if code:
                h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu capture, if it was taken
    on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        e = t[f"{kernel}:{workload}"]
        if e.get("source_hash") == source_hash(kernel):
            return e["dram_bytes_per_launch"]
    except Exception:
        pass
    return None


# ----------------------------------------------------------------- clocks

def smi_id(props, index: int) -> str:
    """nvidia-smi --id for a torch device: its PCI address when known."""
    try:
        return f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
    except Exception:
        return str(index)


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.t is not None:
            self.t.join(timeout=2)

    def summary(self, t0: float, t1: float, strict: bool = False):
        rows = [l for (t, l) in self.lines if t0 - 0.25 <= t <= t1 + 0.25]
        if not rows and not strict:
            rows = [l for (_, l) in self.lines]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            f = [x.strip() for x in r.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------- workloads

class Decode:
    """Decode-shape linear: X[8,5120] bf16 (0.1 % channels x60), W[12288,5120]."""

    def __init__(self, torch, nv, synth, dev, rank, l2_bytes):
        w = synth.DECODE
        self.w = w
        self.torch, self.nv = torch, nv
        x = synth.activation(w, device=dev, seed=w.seed + 1000 * rank)
        wt = synth.weight(w, device=dev)
        am = torch.empty(1, dtype=torch.float32, device=dev)
        nv.nvfp4_amax(x, am)
        self.ga = 2688.0 / am.item()          # static (calibrated) activation scale
        nv.nvfp4_amax(wt, am)
        self.gw = 2688.0 / am.item()
        wc, ws = nv.alloc_quantized(w.N, w.K, dev)
        nv.nvfp4_quantize(wt, self.gw, wc, ws)
        per_copy = wc.numel() + ws.numel()
        self.n_copies = max(2, math.ceil(3 * l2_bytes / per_copy))
        self.w_copies = [(wc, ws)] + [(wc.clone(), ws.clone()) for _ in range(self.n_copies - 1)]
        for c, sc in self.w_copies:            # model weights: read-only while the layer runs
            nv.nvfp4_declare_static(c)
            nv.nvfp4_declare_static(sc)
        self.x = x
        self.a_codes, self.a_sc = nv.alloc_quantized(w.M, w.K, dev)
        self.out = torch.empty(w.M, w.N, dtype=torch.bfloat16, device=dev)
        del wt
        # algorithmic bytes: quantize (X read, codes + scales written) +
        # GEMM (A codes/scales, W codes/scales read, output written)
        M, N, K = w.M, w.N, w.K
        self.gemm_bytes = M * K // 2 + M * K // 16 + N * K // 2 + N * K // 16 + M * N * 2
        self.quant_bytes = M * K * 2 + M * K // 2 + M * K // 16
        self.step_bytes = self.gemm_bytes + self.quant_bytes
        # the whole layer in one kernel: X in, W in, output out (the
        # quantized activation never leaves the chip)
        self.layer_bytes = M * K * 2 + N * K // 2 + N * K // 16 + M * N * 2
        self.launches_per_step = 2

    def gemm_only(self, i):
        w = self.w
        wc, ws = self.w_copies[i % self.n_copies]
        self.nv.nvfp4_gemm(self.a_codes, self.a_sc, self.ga, wc, ws, self.gw, w.M, w.N, w.K, self.out)

    def linear(self, i):
        # the layer through its public call: quantize X into the activation
        # buffers, block-scaled GEMM, dequantizing epilogue (two kernels)
        w = self.w
        wc, ws = self.w_copies[i % self.n_copies]
        self.nv.nvfp4_linear(self.x, self.ga, wc, ws, self.gw, w.N, self.out, self.a_codes, self.a_sc)

    def linear_one_kernel(self, i):
        # the same layer as one kernel that quantizes X in shared memory
        w = self.w
        wc, ws = self.w_copies[i % self.n_copies]
        self.nv.nvfp4_linear(self.x, self.ga, wc, ws, self.gw, w.N, self.out)

    def config(self):
        w = self.w
        return {"workload": "decode-shape linear X[8,5120] bf16 x W[12288,5120] nvfp4 -> bf16",
                "M": w.M, "N": w.N, "K": w.K, "global_batch": w.M,
                "l2": f"weight rotates through {self.n_copies} copies "
                      f"({self.n_copies * (w.N * w.K // 2 + w.N * w.K // 16) / 1e6:.0f} MB > 3x L2)",
                "weights": "declared read-only (nvfp4_declare_static): first stages load before the "
                           "preceding kernel ends"}


class Prefill:
    """Prefill-shape linear: X[32768,5120] heavy-tailed bf16, W[17408,5120]."""

    def __init__(self, torch, nv, synth, dev, rank, l2_bytes, w=None):
        w = synth.PREFILL if w is None else w
        self.w = w
        self.torch, self.nv = torch, nv
        x = synth.activation(w, device=dev, seed=w.seed + 1000 * rank)
        wt = synth.weight(w, device=dev)
        am = torch.empty(1, dtype=torch.float32, device=dev)
        nv.nvfp4_amax(x, am)
        self.ga = 2688.0 / am.item()
        nv.nvfp4_amax(wt, am)
        self.gw = 2688.0 / am.item()
        self.wc, self.ws = nv.alloc_quantized(w.N, w.K, dev)
        nv.nvfp4_quantize(wt, self.gw, self.wc, self.ws)
        torch.cuda.synchronize()
        nv.nvfp4_declare_static(self.wc)       # model weights: read-only while the layer runs
        nv.nvfp4_declare_static(self.ws)
        del wt
        self.x = x
        self.a_codes, self.a_sc = nv.alloc_quantized(w.M, w.K, dev)
        self.out = torch.empty(w.M, w.N, dtype=torch.bfloat16, device=dev)
        M, N, K = w.M, w.N, w.K
        self.flops = 2.0 * M * N * K
        self.launches_per_step = 2

    def step(self, i):
        w = self.w
        self.nv.nvfp4_quantize(self.x, self.ga, self.a_codes, self.a_sc)
        self.nv.nvfp4_gemm(self.a_codes, self.a_sc, self.ga, self.wc, self.ws, self.gw, w.M, w.N, w.K, self.out)

    def gemm_only(self, i):
        w = self.w
        self.nv.nvfp4_gemm(self.a_codes, self.a_sc, self.ga, self.wc, self.ws, self.gw, w.M, w.N, w.K, self.out)


class FusedGDN:
    """Fused GDN in-projection: X[4096,5120]; W segments 8192/4096/48/48."""

    def __init__(self, torch, nv, synth, dev, rank, l2_bytes):
        w = synth.FUSED_GDN
        self.w = w
        self.nv = nv
        x = synth.activation(w, device=dev, seed=w.seed + 1000 * rank)
        wt = synth.weight(w, device=dev)
        self.offs = synth.segment_offsets(w)
        am = torch.empty(1, dtype=torch.float32, device=dev)
        nv.nvfp4_amax(x, am)
        self.ga = 2688.0 / am.item()
        self.gs = []
        rm = torch.empty(w.N, w.K // 16, dtype=torch.uint8, device=dev)
        self.wc = torch.empty(w.N, w.K // 2, dtype=torch.uint8, device=dev)
        for i in range(len(w.segments)):
            seg = wt[self.offs[i]:self.offs[i + 1]].contiguous()
            nv.nvfp4_amax(seg, am)
            g = 2688.0 / am.item()
            self.gs.append(g)
            c, s = nv.alloc_quantized(seg.shape[0], w.K, dev, nv.SF_ROWMAJOR)
            nv.nvfp4_quantize(seg, g, c, s, nv.SF_ROWMAJOR)
            self.wc[self.offs[i]:self.offs[i + 1]] = c
            rm[self.offs[i]:self.offs[i + 1]] = s.view(-1, w.K // 16)
        self.ws = torch.empty(nv.nvfp4_scale_bytes(w.N, w.K), dtype=torch.uint8, device=dev)
        nv.nvfp4_swizzle_scales(rm, w.N, w.K, self.ws)
        torch.cuda.synchronize()
        nv.nvfp4_declare_static(self.wc)       # model weights: read-only while the layer runs
        nv.nvfp4_declare_static(self.ws)
        del wt
        self.x = x
        self.a_codes, self.a_sc = nv.alloc_quantized(w.M, w.K, dev)
        self.out = torch.empty(w.M, w.N, dtype=torch.bfloat16, device=dev)
        self.flops = 2.0 * w.M * w.N * w.K
        self.launches_per_step = 2

    def step(self, i):
        w = self.w
        self.nv.nvfp4_quantize(self.x, self.ga, self.a_codes, self.a_sc)
        self.nv.nvfp4_fused_proj(self.a_codes, self.a_sc, self.ga, self.wc, self.ws, self.offs, self.gs,
                                 w.M, w.K, self.out)


class QuantSweep:
    """One point of the quantize sweep.  Where X is smaller than the L2, the
    step rotates through copies of X (and of the outputs) totalling more
    than 3x the L2 (at most 16 copies), so no step finds its input in L2;
    the M <= 64 points are latency-bound and use at most 16 copies."""

    MAX_COPIES = 16

    def __init__(self, torch, nv, synth, dev, M, K, l2_bytes):
        self.nv = nv
        x = synth.quant_sweep_activation(M, K, device=dev)
        self.M, self.K = M, K
        self.bytes = M * K * 2 + M * K // 2 + M * K // 16
        self.n_copies = max(1, min(self.MAX_COPIES, math.ceil(3 * l2_bytes / self.bytes)))
        self.xs = [x] + [x.clone() for _ in range(self.n_copies - 1)]
        self.outs = [nv.alloc_quantized(M, K, dev) for _ in range(self.n_copies)]
        self.am = torch.empty(1, dtype=torch.float32, device=dev)
        nv.nvfp4_amax(x, self.am)
        self.g = 2688.0 / self.am.item()

    def step(self, i):
        # static global scale (a calibrated deployment): codes and scales only
        j = i % self.n_copies
        codes, sc = self.outs[j]
        self.nv.nvfp4_quantize(self.xs[j], self.g, codes, sc, self.nv.SF_TCGEN05)

    def step_amax(self, i):
        # the same, also reporting the tensor's amax through amax_out
        j = i % self.n_copies
        codes, sc = self.outs[j]
        self.nv.nvfp4_quantize(self.xs[j], self.g, codes, sc, self.nv.SF_TCGEN05, self.am)

    def step_dynamic(self, i):
        # dynamic global scale: the amax pass (K0) then the quantizer (K1),
        # 4.5625 B per element.  The C-ABI takes g on the host, so every step
        # uses the g of the first pass (the same value; the same work)
        j = i % self.n_copies
        codes, sc = self.outs[j]
        self.nv.nvfp4_amax(self.xs[j], self.am)
        self.nv.nvfp4_quantize(self.xs[j], self.g, codes, sc, self.nv.SF_TCGEN05)


# ----------------------------------------------------------------- timing

REPLAYS = 10     # timed replays of each captured graph; the median is reported


def time_graph(torch, fn, steps, warmup, stream, replays=REPLAYS):
    """Warm up eagerly, capture `steps` calls of fn(i) in one CUDA graph and
    replay it once untimed; then replay it `replays` times back to back, each
    replay bracketed by CUDA events on `stream`.  Returns (median over the
    replays of ms per step, graph)."""
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(steps):
            fn(i)
    g.replay()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(replays)]
    for start, end in evs:
        start.record(stream)
        g.replay()
        end.record(stream)
    evs[-1][1].synchronize()
    per_step = sorted(start.elapsed_time(end) / steps for start, end in evs)
    return statistics.median(per_step), g


def time_burst(torch, fn, steps, stream, replays=REPLAYS, idle_s=0.25):
    """Burst regime: a graph of `steps` calls replayed `replays` times with
    the GPU idle for `idle_s` before each timed replay, so every replay starts
    below the power cap.  Returns the median over the replays of ms per step."""
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=stream):
        for i in range(steps):
            fn(i)
    g.replay()
    torch.cuda.synchronize()
    per_step = []
    for _ in range(replays):
        time.sleep(idle_s)
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        g.replay()
        end.record(stream)
        end.synchronize()
        per_step.append(start.elapsed_time(end) / steps)
    del g
    return statistics.median(per_step)


def time_eager(torch, fn, steps, warmup):
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(s)
    for i in range(steps):
        fn(i)
    end.record(s)
    end.synchronize()
    return start.elapsed_time(end) / steps


def soak_clocks(torch, graph, ms_per_replay, stream, sampler, seconds=1.0):
    """Replay a captured graph back to back for about `seconds` (untimed) and
    return the clock samples of that window, or None without samples."""
    if sampler is None or graph is None:
        return None
    n = max(1, int(seconds / max(ms_per_replay * 1e-3, 1e-6)))
    torch.cuda.synchronize()
    t0 = time.time()
    with torch.cuda.stream(stream):
        for _ in range(n):
            graph.replay()
    torch.cuda.synchronize()
    return sampler.summary(t0, time.time(), strict=True)


# ----------------------------------------------------------------- CPU oracle

def oracle_decode_sample(budget_s=12.0, max_steps=40, warmup=0, exact=False):
    """Time the CPU oracle on the decode workload: quantize X + FP64 GEMM.
    warmup untimed steps first; then max_steps timed steps, or (exact=False)
    fewer if budget_s runs out first."""
    import numpy as np
    import torch
    import oracle
    import synth
    w = synth.DECODE
    threads = os.cpu_count() or 1
    oracle.set_threads(threads)
    x = synth.activation(w).float().numpy()
    wt = synth.weight(w).float().numpy()
    gw = oracle.global_scale(oracle.amax(wt))
    wc, wsc = oracle.quantize(wt, gw)
    ga = oracle.global_scale(oracle.amax(x))
    for _ in range(warmup):
        ac, asc = oracle.quantize(x, ga)
        oracle.gemm(ac, asc, ga, wc, wsc, gw)
    times = []
    t_end = time.time() + budget_s
    while len(times) < max_steps and (exact or not times or time.time() < t_end):
        t0 = time.perf_counter()
        ac, asc = oracle.quantize(x, ga)
        oracle.gemm(ac, asc, ga, wc, wsc, gw)
        times.append(time.perf_counter() - t0)
    M, N, K = w.M, w.N, w.K
    step_bytes = (M * K // 2 + M * K // 16 + N * K // 2 + N * K // 16 + M * N * 2) + (M * K * 2 + M * K // 2 + M * K // 16)
    sec = sum(times) / len(times)
    return {"value": step_bytes / sec / 1e9, "unit": "GB/s", "cores": oracle.get_threads(), "kind": "oracle",
            "sample": f"{len(times)} full decode steps (quantize X[8,5120] + FP64 GEMM 8x12288x5120), "
                      f"{sec * 1e3:.1f} ms each"}, len(times), sec


# ----------------------------------------------------------------- ranks

def aggregate_replicas(ms_local: float, units_per_rank: float, world: int, dist=None, device="cpu"):
    """N independent replicas: the job's time is the slowest rank's, and the
    job processed world * units_per_rank units in it.  Returns (ms, units/s)."""
    ms = ms_local
    if dist is not None and world > 1:
        import torch
        t = torch.tensor([ms_local], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    return ms, world * units_per_rank / (ms * 1e-3)


# ----------------------------------------------------------------- main

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    # exactly K timed steps after W untimed ones, each one full decode step of
    # the oracle on the host cores (about 0.1-0.3 s each)
    cpu, n, sec = oracle_decode_sample(max_steps=max(1, args.steps), warmup=args.warmup, exact=True)
    line = {"impl": "reference", "metric": METRIC, "value": cpu["value"], "unit": "GB/s", "n_gpus": args.gpus,
            "steps": n, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None, "dtype": "f64 (GEMM) / f32 (quantize)", "data": "synthetic",
            "config": {"workload": "decode-shape linear X[8,5120] bf16 x W[12288,5120] nvfp4 -> bf16",
                       "M": 8, "N": 12288, "K": 5120, "parallelism": "host cores"},
            "cpu_baseline": cpu,
            "e2e": {"value": cpu["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def measure_decode(torch, nv, synth, dev, rank, world, l2, args, stream, barrier, max_over_ranks, peaks,
                   peak_kind):
    """Headline: the decode-shape linear layer as one step = nvfp4_linear
    (quantize X, block-scaled GEMM, dequantizing epilogue: the quantize
    kernel then the GEMM).  Also timed: the same call in its one-kernel form
    and the GEMM alone."""
    d = Decode(torch, nv, synth, dev, rank, l2)
    torch.cuda.synchronize()
    # soak so the clock sampler sees the GPU under this load before timing
    t_soak = time.time()
    i = 0
    while time.time() - t_soak < args.soak:
        d.linear(i)
        i += 1
        if i % 64 == 0:
            torch.cuda.synchronize()
    barrier()
    with torch.cuda.stream(stream):
        ms_lin, g_lin = time_graph(torch, d.linear, args.steps, args.warmup, stream)
        ms_one, g_one = time_graph(torch, d.linear_one_kernel, args.steps, args.warmup, stream)
        ms_gemm, g_gemm = time_graph(torch, d.gemm_only, args.steps, args.warmup, stream)
    barrier()
    t_end = time.time()
    ms_lin = max_over_ranks(ms_lin)
    ms_one = max_over_ranks(ms_one)
    ms_gemm = max_over_ranks(ms_gemm)
    del g_lin, g_one, g_gemm

    # end to end through the public API: pinned host X in, host result out
    x_host = d.x.cpu().pin_memory()
    out_host = torch.empty(d.out.shape, dtype=d.out.dtype).pin_memory()
    x_dev = torch.empty_like(d.x)

    def e2e_step(i):
        # one C-ABI call: copy X in, the layer, copy the result out
        wc, ws = d.w_copies[i % d.n_copies]
        nv.nvfp4_linear_host(x_host, d.ga, wc, ws, d.gw, d.w.N, out_host, x_dev, d.out, d.a_codes, d.a_sc)

    barrier()
    ms_e2e = max_over_ranks(time_eager(torch, e2e_step, args.steps, args.warmup))
    barrier()

    value = aggregate_replicas(ms_lin, d.step_bytes, world)[1] / 1e9
    gemm_gbs = d.gemm_bytes / (ms_gemm * 1e-3) / 1e9
    hbm_peak = float(peaks["hbm_gbs"])
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_lin, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e2m1, e4m3 block scales, f32 accumulate, bf16 out)",
        "data": "synthetic (seeded; decode X N(0,1) with 0.1% channels x60, W N(0,0.02))",
        "config": dict(d.config(), step="nvfp4_linear: quantize kernel + GEMM kernel (with epilogue)",
                       parallelism=f"replicas x{world}" if world > 1 else "single GPU"),
        "roofline": {"bound": "hbm", "kernel": "nvfp4_gemm_kernel<16,swap>", "achieved": gemm_gbs,
                     "peak": hbm_peak, "unit": "GB/s", "frac": gemm_gbs / hbm_peak,
                     "peak_kind": f"{peak_kind} copy bandwidth",
                     "algorithmic_bytes_per_launch": d.gemm_bytes, "ms_per_launch": ms_gemm,
                     "traffic": profiled_traffic("nvfp4_gemm_kernel", "decode")},
        "e2e": {"value": world * d.step_bytes / (ms_e2e * 1e-3) / 1e9, "unit": "GB/s",
                "ms_per_step": ms_e2e, "h2d_bytes_per_step": d.x.numel() * d.x.element_size(),
                "d2h_bytes_per_step": d.out.numel() * d.out.element_size()},
        "timing": f"median over {REPLAYS} back-to-back replays of a CUDA graph of K steps, CUDA events on the "
                  f"launching stream; every replay is inside the timed region",
        "gpu_launches": d.launches_per_step * args.steps * REPLAYS,
        "decode_one_kernel": {
            "step": "nvfp4_linear without activation buffers: one kernel quantizes X in shared memory",
            "ms_per_step": ms_one, "GB/s": world * d.layer_bytes / (ms_one * 1e-3) / 1e9,
            "bytes_per_step": d.layer_bytes},
    }
    del d
    nv.nvfp4_forget_static()
    return line, t_soak, t_end


SUSTAINED_S = 0.1   # a timed region of back-to-back launches at least this long runs under the power cap


def tensor_roofline(kernel, flops, ms, peaks, peak_kind, traffic, timed_s):
    """Roofline record of a tensor-bound launch against the dense FP4 peak:
    the measured BF16 cuBLAS rate times the nominal FP4 : BF16 ratio, taken
    from the sustained (power-capped) measurement when the launches were timed
    back to back for at least SUSTAINED_S seconds, else from the burst one.
    The other regime's fraction is given beside it."""
    fp4_burst = float(peaks["bf16_tflops"]) * FP4_OVER_BF16
    fp4_sust = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])) * FP4_OVER_BF16
    sustained = timed_s >= SUSTAINED_S
    peak = fp4_sust if sustained else fp4_burst
    tf = flops / (ms * 1e-3) / 1e12
    rec = {"bound": "tensor", "kernel": kernel, "flops_per_launch": flops, "ms_per_launch": ms,
           "regime": f"{'sustained' if sustained else 'burst'} ({timed_s * 1e3:.0f} ms of back-to-back launches)",
           "peak_kind": f"{peak_kind} bf16 cuBLAS {'sustained' if sustained else 'burst'} x {FP4_OVER_BF16:g} "
                        f"(nominal fp4/bf16)",
           "traffic": traffic, "unit": "TFLOP/s"}
    if sustained:
        rec["frac_of_burst_peak"] = round(tf / fp4_burst, 4)
    else:
        rec["frac_of_sustained_peak"] = round(tf / fp4_sust, 4)
    rec.update({"peak": round(peak, 1), "achieved": round(tf, 1), "frac": round(tf / peak, 4)})
    return rec


def measure_prefill(torch, nv, synth, dev, rank, l2, args, stream, peaks, peak_kind, sampler=None):
    w = synth.PREFILL
    if args.prefill_m:
        import dataclasses
        w = dataclasses.replace(w, M=args.prefill_m)
    p = Prefill(torch, nv, synth, dev, rank, l2, w)
    k = max(3, min(args.steps, 20))
    with torch.cuda.stream(stream):
        ms_p, g1 = time_graph(torch, p.step, k, 3, stream)
        ms_pg, g2 = time_graph(torch, p.gemm_only, k, 3, stream)
    clk = soak_clocks(torch, g2, ms_pg * k, stream, sampler)
    del g1, g2
    with torch.cuda.stream(stream):
        ms_burst = time_burst(torch, p.gemm_only, 2, stream)
    traffic = profiled_traffic("nvfp4_gemm_kernel", "prefill")
    res = {
        "workload": f"prefill X[{w.M},5120] x W[17408,5120] nvfp4 -> bf16; inputs 129 MB + 1.14 GB output > L2",
        "step": "quantize + GEMM", "ms_per_step": round(ms_p, 5),
        "step_tflops": round(p.flops / (ms_p * 1e-3) / 1e12, 1),
        "clocks_gemm_back_to_back": clk,
        "roofline_burst": tensor_roofline("nvfp4_gemm_kernel<256>", p.flops, ms_burst, peaks, peak_kind, traffic,
                                          2 * ms_burst * 1e-3),
        "roofline": tensor_roofline("nvfp4_gemm_kernel<256>", p.flops, ms_pg, peaks, peak_kind, traffic,
                                    REPLAYS * k * ms_pg * 1e-3)}
    del p
    nv.nvfp4_forget_static()
    return res


def measure_fused(torch, nv, synth, dev, rank, l2, args, stream, peaks, peak_kind):
    f = FusedGDN(torch, nv, synth, dev, rank, l2)
    k = max(3, min(args.steps, 20))
    w = f.w

    def gemm_only(i):
        f.nv.nvfp4_fused_proj(f.a_codes, f.a_sc, f.ga, f.wc, f.ws, f.offs, f.gs, w.M, w.K, f.out)

    with torch.cuda.stream(stream):
        ms_f, g3 = time_graph(torch, f.step, k, 3, stream)
        ms_g, g4 = time_graph(torch, gemm_only, k, 3, stream)
    del g3, g4
    res = {"workload": "fused GDN projection X[4096,5120] x W[8192|4096|48|48, 5120], per-segment scales",
           "step": "quantize + fused GEMM", "ms_per_step": round(ms_f, 5),
           "step_tflops": round(f.flops / (ms_f * 1e-3) / 1e12, 1),
           "roofline": tensor_roofline("nvfp4_gemm_kernel<256> (segment table)", f.flops, ms_g, peaks, peak_kind,
                                       profiled_traffic("nvfp4_gemm_kernel", "fused"), REPLAYS * k * ms_g * 1e-3)}
    del f
    nv.nvfp4_forget_static()
    return res


def measure_mma_peak(nv, dev):
    """The device's dense FP4 MMA throughput (context for the tensor
    rooflines; the rooflines keep the measured BF16 x 4 denominator)."""
    tf, per_clk = nv.nvfp4_measure_mma_peak(5000, dev)
    return {"kernel": "mma_peak_kernel: 148 CTAs x 20,000 back-to-back tcgen05.mma kind::mxf4nvf4 "
                      "128x256x64 from shared memory",
            "TFLOP/s": round(tf, 1), "flop_per_clk_per_sm": round(per_clk, 1),
            "at_1965_MHz_TFLOP/s": round(per_clk * 148 * 1.965e9 / 1e12, 1)}


def measure_quant_sweep(torch, nv, synth, dev, args, stream, peaks, l2):
    hbm_peak = float(peaks["hbm_gbs"])
    sweep = {}
    for M in synth.QUANT_SWEEP_M:
        for K in synth.QUANT_SWEEP_K:
            if args.quant_point and args.quant_point != f"{M}x{K}":
                continue
            q = QuantSweep(torch, nv, synth, dev, M, K, l2)
            kk = max(3, min(args.steps, 50))
            with torch.cuda.stream(stream):
                ms_q, g4 = time_graph(torch, q.step, kk, 3, stream)
                del g4
                ms_a, g5 = time_graph(torch, q.step_amax, kk, 3, stream)
                del g5
                ms_d, g6 = time_graph(torch, q.step_dynamic, kk, 3, stream)
                del g6
            gbs = q.bytes / (ms_q * 1e-3) / 1e9
            dyn_gbs = (q.bytes + 2 * M * K) / (ms_d * 1e-3) / 1e9
            sweep[f"{M}x{K}"] = {"us": round(ms_q * 1e3, 3), "GB/s": round(gbs, 1),
                                 "frac_hbm": round(gbs / hbm_peak, 4), "x_copies": q.n_copies,
                                 "us_with_amax_out": round(ms_a * 1e3, 3),
                                 "us_dynamic_k0_k1": round(ms_d * 1e3, 3),
                                 "frac_hbm_dynamic": round(dyn_gbs / hbm_peak, 4)}
            del q
    return sweep


def measure_calibration(torch, nv, synth, dev, args, stream, peaks):
    """Static calibration: running amax over the calibration batches (one pass
    = CALIB_BATCHES batches), then the static-scale quantization of a held-out
    batch with larger outliers.  Two alternating batch sets and four held-out
    copies keep every pass's inputs out of L2."""
    hbm_peak = float(peaks["hbm_gbs"])
    M, K, nb = synth.CALIB_M, synth.CALIB_K, synth.CALIB_BATCHES
    sets = [[synth.calibration_batch(i + nb * j, M, K, device=dev) for i in range(nb)] for j in range(2)]
    run = torch.empty(2, dtype=torch.float32, device=dev)

    def amax_pass(i):
        r = run[i % 2:i % 2 + 1]
        nv.nvfp4_amax(sets[i % 2][0], r)
        for b in sets[i % 2][1:]:
            nv.nvfp4_amax_accumulate(b, r)

    kk = max(3, min(args.steps, 50))
    with torch.cuda.stream(stream):
        ms_a, g1 = time_graph(torch, amax_pass, kk, 3, stream)
    del g1
    torch.cuda.synchronize()
    g_static = 2688.0 / float(run[0].item())
    held = synth.held_out_batch(M, K, device=dev)
    copies = [held] + [held.clone() for _ in range(3)]
    codes, sc = nv.alloc_quantized(M, K, dev)

    def quant(i):
        nv.nvfp4_quantize(copies[i % 4], g_static, codes, sc)

    with torch.cuda.stream(stream):
        ms_q, g2 = time_graph(torch, quant, kk, 3, stream)
    del g2
    torch.cuda.synchronize()
    held_sat = int((sc == 0x7E).sum().item())
    cal_codes, cal_sc = nv.alloc_quantized(M, K, dev)
    nv.nvfp4_quantize(sets[0][0], g_static, cal_codes, cal_sc)
    torch.cuda.synchronize()
    cal_sat = int((cal_sc == 0x7E).sum().item())
    pass_bytes = nb * M * K * 2
    q_bytes = M * K * 2 + M * K // 2 + M * K // 16
    res = {"workload": f"{nb} calibration batches X[{M},{K}] bf16 (outliers 48x RMS), then a held-out "
                       f"batch (368x RMS) quantized with the static scale",
           "amax_pass_us": ms_a * 1e3, "amax_GB/s": pass_bytes / (ms_a * 1e-3) / 1e9,
           "amax_frac_hbm": pass_bytes / (ms_a * 1e-3) / 1e9 / hbm_peak,
           "static_quant_us": ms_q * 1e3, "static_quant_GB/s": q_bytes / (ms_q * 1e-3) / 1e9,
           "static_quant_frac_hbm": q_bytes / (ms_q * 1e-3) / 1e9 / hbm_peak,
           "scale_bytes_at_448": {"held_out": held_sat, "calibration_batch_0": cal_sat},
           "launches_per_pass": nb}
    del sets, copies, codes, sc
    return res


def measure_harmonize(torch, nv, synth, dev, rank, l2, args, stream, peaks):
    """Offline scale harmonisation of the fused GDN weight (TCGEN05 scales)
    to g = min g_i, timed over enough scale copies to exceed L2; then the
    single-scale GEMM on the harmonized scales and the unrepaired single-
    scale GEMM, each compared per segment with the exact per-segment
    epilogue (relative Frobenius error)."""
    hbm_peak = float(peaks["hbm_gbs"])
    f = FusedGDN(torch, nv, synth, dev, rank, l2)
    w = f.w
    g = min(f.gs)
    n_bytes = f.ws.numel()
    n_copies = max(2, math.ceil(3 * l2 / (2 * n_bytes)))
    srcs = [f.ws] + [f.ws.clone() for _ in range(n_copies - 1)]
    dsts = [torch.empty_like(f.ws) for _ in range(n_copies)]

    def harm(i):
        nv.nvfp4_harmonize_scales(srcs[i % n_copies], w.N, w.K, f.offs, f.gs, g, dsts[i % n_copies])

    kk = max(3, min(args.steps, 50))
    with torch.cuda.stream(stream):
        ms_h, g1 = time_graph(torch, harm, kk, 3, stream)
    del g1
    f.step(0)
    exact = torch.empty(w.M, w.N, dtype=torch.float32, device=dev)
    nv.nvfp4_fused_proj(f.a_codes, f.a_sc, f.ga, f.wc, f.ws, f.offs, f.gs, w.M, w.K, exact)
    harmonized = torch.empty_like(exact)
    nv.nvfp4_gemm(f.a_codes, f.a_sc, f.ga, f.wc, dsts[0], g, w.M, w.N, w.K, harmonized)
    single = torch.empty_like(exact)
    nv.nvfp4_gemm(f.a_codes, f.a_sc, f.ga, f.wc, f.ws, f.gs[0], w.M, w.N, w.K, single)
    torch.cuda.synchronize()

    def seg_err(o):
        out = []
        for i in range(len(f.gs)):
            a, b = o[:, f.offs[i]:f.offs[i + 1]].double(), exact[:, f.offs[i]:f.offs[i + 1]].double()
            out.append(float((a - b).norm() / b.norm()))
        return out

    byts = 2 * n_bytes
    res = {"workload": f"fused GDN weight scales [{w.N}, {w.K // 16}] TCGEN05 ({n_bytes} B), segments "
                       f"{list(w.segments)}, to g = min g_i",
           "us": ms_h * 1e3, "GB/s": byts / (ms_h * 1e-3) / 1e9, "frac_hbm": byts / (ms_h * 1e-3) / 1e9 / hbm_peak,
           "g_ratio": [g / x for x in f.gs],
           "seg_rel_fro_harmonized": seg_err(harmonized),
           "seg_rel_fro_single_scale_unrepaired": seg_err(single)}
    del f, srcs, dsts
    nv.nvfp4_forget_static()
    return res


def measure_mx(torch, nv, synth, dev, rank, l2, args, stream, peaks, peak_kind, sampler=None):
    """MXFP4, the contrast format: its quantizer (X[4096,5120] bf16), its
    kind::mxf4 GEMM on the prefill and decode shapes (weights rotated through
    copies larger than L2), and the GEMM error of NVFP4 and MXFP4 against the
    FP64 product of the unquantized operands, on the prefill activation
    recipe (outlier channels at 63x RMS)."""
    hbm_peak = float(peaks["hbm_gbs"])
    tc_peak = float(peaks["bf16_tflops"]) * FP4_OVER_BF16
    res = {}
    kk = max(3, min(args.steps, 50))
    # quantizer
    M, K = 4096, 5120
    xs = [synth.activation(synth.PREFILL, device=dev, M=M, seed=synth.PREFILL.seed + 1000 * rank)]
    xs += [xs[0].clone() for _ in range(3)]
    qc, qs = nv.alloc_mx_quantized(M, K, dev)

    def q(i):
        nv.nvfp4_mx_quantize(xs[i % 4], qc, qs)

    with torch.cuda.stream(stream):
        ms_q, g1 = time_graph(torch, q, kk, 3, stream)
    del g1
    qb = M * K * 2 + M * K // 2 + M * K // 32
    res["quantize_4096x5120"] = {"us": ms_q * 1e3, "GB/s": qb / (ms_q * 1e-3) / 1e9,
                                 "frac_hbm": qb / (ms_q * 1e-3) / 1e9 / hbm_peak}
    # prefill-shape GEMM
    w = synth.PREFILL
    pm = args.prefill_m or w.M
    x = synth.activation(w, device=dev, M=pm, seed=w.seed + 1000 * rank)
    wt = synth.weight(w, device=dev)
    ac, as_ = nv.alloc_mx_quantized(pm, w.K, dev)
    wc, ws = nv.alloc_mx_quantized(w.N, w.K, dev)
    nv.nvfp4_mx_quantize(x, ac, as_)
    nv.nvfp4_mx_quantize(wt, wc, ws)
    del x, wt
    out = torch.empty(pm, w.N, dtype=torch.bfloat16, device=dev)

    def gp(i):
        nv.nvfp4_mx_gemm(ac, as_, wc, ws, pm, w.N, w.K, out)

    kp = max(3, min(args.steps, 10))
    with torch.cuda.stream(stream):
        ms_p, g2 = time_graph(torch, gp, kp, 3, stream)
    clk = soak_clocks(torch, g2, ms_p * kp, stream, sampler)
    del g2
    fl = 2.0 * pm * w.N * w.K
    res["gemm_prefill"] = {"shape": [pm, w.N, w.K], "ms": ms_p, "TFLOP/s": fl / (ms_p * 1e-3) / 1e12,
                           "frac_fp4_peak": fl / (ms_p * 1e-3) / 1e12 / tc_peak, "peak": peak_kind,
                           "clocks_gemm_back_to_back": clk}
    del ac, as_, wc, ws, out
    # decode-shape GEMM
    d = synth.DECODE
    x = synth.activation(d, device=dev, seed=d.seed + 1000 * rank)
    wt = synth.weight(d, device=dev)
    ac, as_ = nv.alloc_mx_quantized(d.M, d.K, dev)
    nv.nvfp4_mx_quantize(x, ac, as_)
    wc, ws = nv.alloc_mx_quantized(d.N, d.K, dev)
    nv.nvfp4_mx_quantize(wt, wc, ws)
    per = wc.numel() + ws.numel()
    n_copies = max(2, math.ceil(3 * l2 / per))
    copies = [(wc, ws)] + [(wc.clone(), ws.clone()) for _ in range(n_copies - 1)]
    out = torch.empty(d.M, d.N, dtype=torch.bfloat16, device=dev)

    def gd(i):
        c, s_ = copies[i % n_copies]
        nv.nvfp4_mx_gemm(ac, as_, c, s_, d.M, d.N, d.K, out)

    with torch.cuda.stream(stream):
        ms_d, g3 = time_graph(torch, gd, kk, 3, stream)
    del g3
    db = ac.numel() + as_.numel() + per + d.M * d.N * 2
    res["gemm_decode"] = {"shape": [d.M, d.N, d.K], "us": ms_d * 1e3, "GB/s": db / (ms_d * 1e-3) / 1e9,
                          "frac_hbm": db / (ms_d * 1e-3) / 1e9 / hbm_peak}
    del copies, wc, ws, ac, as_, x, wt
    # accuracy against the FP64 product of the unquantized operands
    M, N, K = 4096, 4096, w.K
    x = synth.activation(w, device=dev, M=M)
    wt = synth.weight(w, device=dev, N=N)
    ref = x.double() @ wt.double().T
    am = torch.empty(1, dtype=torch.float32, device=dev)
    nv.nvfp4_amax(x, am)
    ga = 2688.0 / am.item()
    nv.nvfp4_amax(wt, am)
    gw = 2688.0 / am.item()
    a_c, a_s = nv.alloc_quantized(M, K, dev)
    w_c, w_s = nv.alloc_quantized(N, K, dev)
    nv.nvfp4_quantize(x, ga, a_c, a_s)
    nv.nvfp4_quantize(wt, gw, w_c, w_s)
    o_nv = torch.empty(M, N, dtype=torch.float32, device=dev)
    nv.nvfp4_gemm(a_c, a_s, ga, w_c, w_s, gw, M, N, K, o_nv)
    ma, mas = nv.alloc_mx_quantized(M, K, dev)
    mw, mws = nv.alloc_mx_quantized(N, K, dev)
    nv.nvfp4_mx_quantize(x, ma, mas)
    nv.nvfp4_mx_quantize(wt, mw, mws)
    o_mx = torch.empty_like(o_nv)
    nv.nvfp4_mx_gemm(ma, mas, mw, mws, M, N, K, o_mx)
    torch.cuda.synchronize()
    res["gemm_rel_fro_vs_unquantized"] = {
        "workload": f"X[{M},{K}] prefill recipe x W[{N},{K}] N(0,0.02)",
        "nvfp4": float((o_nv.double() - ref).norm() / ref.norm()),
        "mxfp4": float((o_mx.double() - ref).norm() / ref.norm())}
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--only", default="all", choices=["all", "decode", "prefill", "fused", "quant", "calib", "harmonize", "mx",
                                                      "peak"])
    ap.add_argument("--prefill-m", type=int, default=0, help="override M of the prefill workload")
    ap.add_argument("--soak", type=float, default=1.0, help="seconds of untimed decode steps first")
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--quant-point", default="", help="MxK: run only this point of the quantize sweep")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import nvfp4_w4a4_quantized_10_b200 as nv
    import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist

    def barrier():
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(v: float) -> float:
        return aggregate_replicas(v, 0.0, world, pg, dev)[0]

    peaks, peak_kind = load_peaks()
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 * 1024 * 1024) or 126 * 1024 * 1024
    sampler = ClockSampler(smi_id(props, local))
    sampler.start()
    stream = torch.cuda.Stream(device=dev)

    if args.only != "all" and world == 1:
        if args.only == "decode":
            res, _, _ = measure_decode(torch, nv, synth, dev, rank, world, l2, args, stream, barrier,
                                       max_over_ranks, peaks, peak_kind)
        elif args.only == "prefill":
            res = measure_prefill(torch, nv, synth, dev, rank, l2, args, stream, peaks, peak_kind, sampler)
        elif args.only == "fused":
            res = measure_fused(torch, nv, synth, dev, rank, l2, args, stream, peaks, peak_kind)
        elif args.only == "calib":
            res = measure_calibration(torch, nv, synth, dev, args, stream, peaks)
        elif args.only == "harmonize":
            res = measure_harmonize(torch, nv, synth, dev, rank, l2, args, stream, peaks)
        elif args.only == "mx":
            res = measure_mx(torch, nv, synth, dev, rank, l2, args, stream, peaks, peak_kind, sampler)
        elif args.only == "peak":
            res = measure_mma_peak(nv, dev)
        else:
            res = measure_quant_sweep(torch, nv, synth, dev, args, stream, peaks, l2)
        sampler.stop()
        print(json.dumps({"only": args.only, "result": res}))
        return 0

    line, t_soak, t_end = measure_decode(torch, nv, synth, dev, rank, world, l2, args, stream, barrier,
                                         max_over_ranks, peaks, peak_kind)
    clk = sampler.summary(t_soak, t_end)
    if clk is not None:
        line["clocks"] = clk
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu, _, _ = oracle_decode_sample()
        line["cpu_baseline"] = cpu
    if not args.no_extra and world == 1:
        def leg(fn, *a):
            # an extra workload that raises is reported as such; the headline
            # line above is already measured and still gets printed
            try:
                return fn(*a)
            except Exception as e:  # noqa: BLE001
                nv.nvfp4_forget_static()
                return {"error": f"{type(e).__name__}: {e}"[:400]}

        # the tensor-bound rows come last, so that the end of the printed
        # line (what a log tail keeps) carries them
        extra = {}
        extra["fp4_mma_peak"] = leg(measure_mma_peak, nv, dev)
        extra["mxfp4"] = leg(measure_mx, torch, nv, synth, dev, rank, l2, args, stream, peaks, peak_kind, sampler)
        extra["harmonize"] = leg(measure_harmonize, torch, nv, synth, dev, rank, l2, args, stream, peaks)
        extra["static_calibration"] = leg(measure_calibration, torch, nv, synth, dev, args, stream, peaks)
        extra["quantize_sweep"] = leg(measure_quant_sweep, torch, nv, synth, dev, args, stream, peaks, l2)
        extra["fused_gdn"] = leg(measure_fused, torch, nv, synth, dev, rank, l2, args, stream, peaks, peak_kind)
        extra["prefill"] = leg(measure_prefill, torch, nv, synth, dev, rank, l2, args, stream, peaks, peak_kind,
                               sampler)
        line["extra"] = extra
    sampler.stop()
    if rank == 0:
        print(json.dumps(line))
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
