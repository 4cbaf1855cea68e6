"""Benchmark: bf16 GEMM TFLOP/s at 8192^3 on B200 (C = A.B, bf16 in, fp32 accumulate and out).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload square8192|square4096|ragged|skinny1000|skinny16|mxfp8_8192|fused8192
                                |fused8192_tanh]
                    [--shape M N K] [--config auto|1cta_128x128|1cta_128x256|2cta_256x256]
                    [--no-configs] [--config-steps S]

One step = one library call over the whole M x N x K problem with the inputs
resident in HBM.  Multi-GPU runs (torchrun, one process per GPU) are
independent replicas: every rank multiplies its own seeded matrices, no data
crosses GPUs, and value = FLOPs of all ranks / the slowest rank's time.

Printed (rank 0): one JSON line with the metric, the device-timed value,
`e2e` (the same metric through the C ABI with host buffers, copies inside
the timed region), `roofline` of the GEMM kernel, `cpu_baseline` (the CPU
oracle on a bounded sample of the same workload), clocks sampled during the
timed region and the number of kernel launches.  The default run (8192^3,
one GPU) adds `configs`: every other configuration's workload timed on its
own after the headline (median, p90, TFLOP/s, GB/s, and the roofline, the
larger of FLOPs / tensor peak and minimum bytes / HBM bandwidth), plus the
single tile's CUDA-graph replay time.  `--impl reference` times the oracle
alone, as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "bf16 GEMM TFLOP/s at 8192³ on 1 B200 (fraction of dense BF16 tensor peak)"
METRIC_MXFP8 = "MXFP8 block-scaled GEMM TFLOP/s at 8192³ on 1 B200"
METRIC_FUSED = "bf16 GEMM + bias + GELU (fused epilogue, bf16 out) TFLOP/s at 8192³ on 1 B200"
UNIT = "TFLOP/s"

# name: (M, N, K, kind, distribution, workload id, description)
WORKLOADS = {
    "square8192": (8192, 8192, 8192, "bf16", "uniform", 3,
                   "gemm 8192x8192x8192, bf16 U[-1,1] in, fp32 accumulate + out"),
    "single_tile128": (128, 128, 128, "bf16", "uniform", 1, "gemm 128x128x128, bf16 U[-1,1] in, fp32 out"),
    "square4096": (4096, 4096, 4096, "bf16", "normal_scaled", 2,
                   "gemm 4096x4096x4096, bf16 N(0,1)/sqrt(K) in, fp32 out"),
    "square4096_bf16": (4096, 4096, 4096, "bf16", "normal_scaled", 2,
                        "gemm 4096x4096x4096, bf16 N(0,1)/sqrt(K) in, bf16 out"),
    "ragged": (4000, 3000, 2000, "bf16", "normal", 4, "gemm 4000x3000x2000, bf16 N(0,1) in, fp32 out"),
    "skinny1000": (1000, 8192, 8192, "bf16", "normal", 5, "gemm 1000x8192x8192, bf16 N(0,1) in, fp32 out"),
    "skinny16": (16, 8192, 8192, "bf16", "normal", 6, "gemm 16x8192x8192, bf16 N(0,1) in, fp32 out"),
    "mxfp8_8192": (8192, 8192, 8192, "mxfp8", "uniform", 8,
                   "block-scaled gemm 8192^3, E4M3 U[-1,1], E8M0 per 32 (exp U{-4..4}), bf16 out"),
    "fused8192": (8192, 8192, 8192, "fused", "uniform", 3,
                  "gelu(A.B + bias) 8192^3, bf16 U[-1,1] in, bias N(0,1) fp32, fp32 accumulate, bf16 out"),
    "fused8192_tanh": (8192, 8192, 8192, "fused", "uniform", 3,
                       "gelu_tanh(A.B + bias) 8192^3 (tanh form of GELU), bf16 U[-1,1] in, bias N(0,1) fp32, "
                       "fp32 accumulate, bf16 out"),
}
# activation of the fused workloads (gemm_bf16_fused's act)
FUSED_ACT = {"fused8192": "gelu", "fused8192_tanh": "gelu_tanh"}
# plain GEMM workloads that write bf16 C (the others write fp32)
BF16_OUT = {"square4096_bf16"}
# the per-config report of the default run: every workload of the five
# configurations, each timed on its own (the headline is the main line)
CONFIG_SET = ("single_tile128", "square4096", "square4096_bf16", "ragged", "skinny1000", "skinny16",
              "mxfp8_8192")

L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_OVER_BF16 = 2.0          # nominal dense ratio (4.5 / 2.25 PFLOP/s)
# nominal B200 figures the fraction is also reported against
NOMINAL = {"bf16_tflops": 2250.0, "hbm_gbs": 8000.0}


def roofline_of(flops: float, min_bytes: float, seconds: float, tensor_tflops: float, hbm_gbs: float) -> dict:
    """The roofline of one launch: its time can be no lower than the larger
    of (FLOPs / tensor peak) and (minimum bytes / HBM bandwidth); that larger
    term names the bound, and frac = roofline time / measured time, which
    equals achieved / peak in the bound's own unit."""
    t_tensor = flops / (tensor_tflops * 1e12)
    t_hbm = min_bytes / (hbm_gbs * 1e9)
    if t_tensor >= t_hbm:
        return {"bound": "tensor", "achieved": flops / seconds / 1e12, "peak": tensor_tflops, "unit": "TFLOP/s",
                "frac": t_tensor / seconds, "roofline_us": t_tensor * 1e6}
    return {"bound": "hbm", "achieved": min_bytes / seconds / 1e9, "peak": hbm_gbs, "unit": "GB/s",
            "frac": t_hbm / seconds, "roofline_us": t_hbm * 1e6}


# The device sources each kernel is compiled from; an ncu traffic figure is
# valid only while these files are unchanged.
KERNEL_SOURCES = {
    "bf16": ["ptx.cuh", "epilogue.cuh", "gemm_bf16_sm100.cuh"],
    "skinny": ["ptx.cuh", "epilogue.cuh", "gemm_bf16_sm100.cuh", "gemm_bf16_skinny_sm100.cuh"],
    "mxfp8": ["ptx.cuh", "epilogue.cuh", "gemm_bf16_sm100.cuh", "gemm_mxfp8_sm100.cuh"],
}


def code_only(text: str) -> str:
    """C++ source without comments and blank lines: an edit to a comment
    leaves the compiled kernel, and so its ncu counters, as they were.
    (The kernel sources hold no '//' or '/*' inside string literals.)"""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def kernel_source_hash(kernel: str = "bf16") -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "dense_gemm_engineering_bf16_b200", "csrc", name), encoding="utf-8") as f:
            h.update(code_only(f.read()).encode())
    return h.hexdigest()[:16]


def kernel_family(config_name: str) -> str:
    if config_name.startswith("mxfp8"):
        return "mxfp8"
    return "skinny" if config_name == "skinny" else "bf16"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def profile_traffic(workload: str, config_name: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources; else None."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    entry = t.get(f"{workload}:{config_name}")
    if not entry or entry.get("kernel_source_hash") != kernel_source_hash(kernel_family(config_name)):
        return None
    return entry.get("dram_bytes_per_launch")


# ------------------------------------------------------------ multi-rank --

def max_over_ranks(x: float, world: int, device=None) -> float:
    """The maximum of x over all ranks (x itself when world == 1)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_step: float, steps: int, world: int, slowest_ms: float) -> float:
    """Replicas: every rank did `steps` steps; the job took the slowest rank's time."""
    return world * steps * flops_per_step / (slowest_ms * 1e-3) / 1e12


class ClockSampler:
    """nvidia-smi clock / throttle samples every 100 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.gpu_id is not None:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return
        time.sleep(0.15)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        return summarize_clocks(self.lines)


def summarize_clocks(lines):
    """Median SM clock, max clock, median power and the throttle reasons seen."""
    sm, smax, power, reasons = [], [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for line in lines:
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            smax.append(float(parts[2]))
            power.append(float(parts[3]))
        except ValueError:
            continue
        for name, val in zip(names, parts[5:9]):
            if val.lower() == "active":
                reasons.add(name)
    if not sm:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
    # "under load": samples drawing at least 60 % of the highest power seen
    # (the sampler brackets the timed region by a few hundred ms of idle)
    pmax = max(power)
    loaded = [i for i, pw in enumerate(power) if pw >= 0.6 * pmax] or list(range(len(sm)))
    return {"sm_mhz": statistics.median(sm[i] for i in loaded), "sm_max_mhz": max(smax),
            "reasons": sorted(reasons), "samples": len(sm), "samples_under_load": len(loaded),
            "power_w_median_under_load": statistics.median(power[i] for i in loaded)}


# -------------------------------------------------------------- workloads --

class Problem:
    """Host operands of one workload and the library call that runs it."""

    def __init__(self, name, shape, rank):
        from dense_gemm_engineering_bf16_b200 import synth
        M, N, K, kind, dist, wid, desc = WORKLOADS[name]
        if shape:
            M, N, K = shape
            dist, wid = "uniform", 90
            desc = {"bf16": f"gemm {M}x{N}x{K}, bf16 U[-1,1] in, fp32 out",
                    "fused": f"gelu(A.B + bias) {M}x{N}x{K}, bf16 U[-1,1] in, bf16 out",
                    "mxfp8": f"block-scaled gemm {M}x{N}x{K}, E4M3 U[-1,1], E8M0 per 32, bf16 out"}[kind]
        self.name, self.M, self.N, self.K, self.kind, self.desc = name, M, N, K, kind, desc
        self.bf16_out = name in BF16_OUT
        self.act = FUSED_ACT.get(name, "gelu")
        self.flops = 2.0 * M * N * K
        if kind == "bf16":
            self.a, self.b = synth.bf16_operands(M, N, K, dist, workload=wid, base=rank)
            self.host = [self.a, self.b]
            self.in_bytes = 2 * (M * K + N * K)
            self.out_bytes = (2 if self.bf16_out else 4) * M * N
        elif kind == "fused":
            self.a, self.b = synth.bf16_operands(M, N, K, dist, workload=wid, base=rank)
            self.bias = synth.normal(synth.derive_seed(wid, 4, rank), (N,)).astype(np.float32)
            self.host = [self.a, self.b, self.bias]
            self.in_bytes = 2 * (M * K + N * K) + 4 * N
            self.out_bytes = 2 * M * N
        else:
            self.a, self.sfa, self.b, self.sfb = synth.mxfp8_operands(M, N, K, workload=wid, base=rank)
            self.host = [self.a, self.sfa, self.b, self.sfb]
            self.in_bytes = M * K + N * K + (M + N) * (K // 32)
            self.out_bytes = 2 * M * N

    def device_arrays(self, torch):
        if self.kind == "bf16":
            return [torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16) for x in self.host]
        if self.kind == "fused":
            return [torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16) for x in self.host[:2]] + \
                [torch.from_numpy(self.bias).cuda()]
        return [torch.from_numpy(np.ascontiguousarray(x)).cuda() for x in self.host]

    def empty_out(self, torch, pinned=False):
        dt = torch.float32 if self.kind == "bf16" and not self.bf16_out else torch.bfloat16
        if pinned:
            return torch.empty((self.M, self.N), dtype=dt).pin_memory()
        return torch.empty((self.M, self.N), dtype=dt, device="cuda")

    def call(self, G, dev, C, stream):
        M, N, K = self.M, self.N, self.K
        if self.kind == "bf16":
            A, B = dev
            G.gemm_bf16(A, B, C, M, N, K, K, K, N, G.OUT_BF16 if self.bf16_out else G.OUT_F32, stream=stream)
        elif self.kind == "fused":
            A, B, bias = dev
            G.gemm_bf16_fused(A, B, C, M, N, K, K, K, N, G.OUT_BF16, G.KMAJOR, G.KMAJOR, 1.0, 0.0, bias,
                              act_code(G, self.act), stream=stream)
        else:
            A, SA, B, SB = dev
            G.gemm_mxfp8(A, SA, B, SB, C, M, N, K, K, K, N, stream=stream)

    def launches(self, G):
        return G.gemm_launches_per_call(self.M, self.N, self.K, self.kind == "mxfp8")

    def oracle_rows(self, rows):
        import oracle
        if self.kind == "bf16":
            return oracle.gemm_bf16_f64(self.a[:rows], self.b, K=self.K)
        if self.kind == "fused":
            c = oracle.gemm_bf16_f64(self.a[:rows], self.b, K=self.K)
            return oracle.epilogue(c, None, 1.0, 0.0, self.bias.astype(np.float64),
                                   {"gelu": oracle.ACT_GELU, "gelu_tanh": oracle.ACT_GELU_TANH}[self.act])
        return oracle.gemm_mxfp8_f64(self.a[:rows], self.sfa[:rows], self.b, self.sfb, K=self.K)


def act_code(G, name: str) -> int:
    return {"gelu": G.ACT_GELU, "gelu_tanh": G.ACT_GELU_TANH}[name]


def fusion_comparison(p, G, dev, torch, stream, steps):
    """The unfused form of the fused workload, timed beside it: a plain GEMM
    writing the bf16 intermediate, then a separate pass C = act(C + bias)
    that reads it back and writes it again.  Fusion saves that pass's two
    intermediate-sized transfers ("GPU 执行模型", section "Fusion 的收益与
    上限": about 2 x the intermediate's bytes).  The fused call, the plain
    GEMM and the pass are interleaved step by step, so all three see the
    same clocks; medians are reported."""
    A, B, bias = dev
    M, N, K = p.M, p.N, p.K
    C1 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    C2 = torch.empty_like(C1)

    act = act_code(G, p.act)

    def fused():
        G.gemm_bf16_fused(A, B, C1, M, N, K, K, K, N, G.OUT_BF16, G.KMAJOR, G.KMAJOR, 1.0, 0.0, bias,
                          act, stream=stream)

    def gemm():
        G.gemm_bf16(A, B, C2, M, N, K, K, K, N, G.OUT_BF16, stream=stream)

    def pointwise():
        G.gemm_bf16_fused(A, B, C2, M, N, 0, K, K, N, G.OUT_BF16, G.KMAJOR, G.KMAJOR, 1.0, 1.0, bias,
                          act, stream=stream)

    for _ in range(3):
        fused(), gemm(), pointwise()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for e in ev:
        e[0].record(stream)
        fused()
        e[1].record(stream)
        gemm()
        e[2].record(stream)
        pointwise()
        e[3].record(stream)
    torch.cuda.synchronize()
    G.gemm_check_device_status(stream)
    med = lambda i: statistics.median(e[i].elapsed_time(e[i + 1]) for e in ev)  # noqa: E731
    fused_ms, gemm_ms, pass_ms = med(0), med(1), med(2)
    inter = 2 * M * N                       # the bf16 intermediate, bytes
    return {"fused_ms": fused_ms, "unfused_gemm_ms": gemm_ms, "unfused_pass_ms": pass_ms,
            "unfused_ms": gemm_ms + pass_ms, "saved_ms": gemm_ms + pass_ms - fused_ms,
            "fused_over_plain_gemm_ms": fused_ms - gemm_ms,
            "ledger_saved_bytes": 2 * inter,
            "unfused_pass_gbs": (2 * inter + 4 * N) / (pass_ms * 1e-3) / 1e9, "steps": steps}


def min_bytes(p: Problem) -> int:
    """Operands read once plus C written once: the byte floor of one call."""
    return p.in_bytes + p.out_bytes


def flush_l2(scratch, clean: bool = True):
    """Evict L2 before a timed call: write a buffer twice the L2's size; with
    `clean`, read it back too, so that the write-backs of the dirty lines the
    write leaves behind happen here, outside the timed events, instead of
    inside the next call (which would then pay for the flush's own traffic)."""
    scratch.zero_()
    if clean:
        scratch.sum()


def time_steps(p: Problem, G, dev, C, torch, stream, steps: int, scratch=None, clean: bool = True):
    """Device time of each of `steps` calls (ms).  With `scratch`, L2 is
    flushed (flush_l2) before every call, outside the events."""
    if scratch is not None:
        ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        for i in range(steps):
            flush_l2(scratch, clean)
            ev_s[i].record(stream)
            p.call(G, dev, C, stream)
            ev_e[i].record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in zip(ev_s, ev_e)], None
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    ev[0].record(stream)
    for i in range(steps):
        p.call(G, dev, C, stream)
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    return [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)], ev[0].elapsed_time(ev[-1])


def graph_replay_us(p: Problem, G, dev, C, torch, stream, steps: int, scratch) -> float:
    """Median device time (us) of one call captured in a CUDA graph and
    replayed, L2 flushed before each replay outside the events."""
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()              # capture needs a stream other than the default one
    side.wait_stream(stream)
    with torch.cuda.graph(g, stream=side):
        p.call(G, dev, C, side)
    stream.wait_stream(side)
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for i in range(steps):
        flush_l2(scratch)
        ev_s[i].record(stream)
        g.replay()
        ev_e[i].record(stream)
    torch.cuda.synchronize()
    t = statistics.median(a.elapsed_time(b) for a, b in zip(ev_s, ev_e)) * 1e3
    del g
    return t


def config_report(G, torch, stream, peaks: dict, steps: int, warmup: int) -> dict:
    """Every workload of CONFIG_SET timed on its own, on the same GPU, with
    the same L2 rule as the headline: median and p90 of `steps` calls,
    TFLOP/s and GB/s at the median, and the roofline (the larger of FLOPs /
    tensor peak and minimum bytes / HBM bandwidth) against the measured
    peaks and against the nominal B200 figures."""
    scratch = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda")
    out = {}
    for name in CONFIG_SET:
        p = Problem(name, None, 0)
        dev = p.device_arrays(torch)
        C = p.empty_out(torch)
        for _ in range(warmup):
            p.call(G, dev, C, stream)
        G.gemm_check_device_status(stream)
        flush = needs_l2_flush(min_bytes(p))
        per_step, _ = time_steps(p, G, dev, C, torch, stream, steps, scratch if flush else None)
        # the same with the write-only flush: L2 left full of dirty lines
        dirty = time_steps(p, G, dev, C, torch, stream, steps, scratch, clean=False)[0] if flush else None
        G.gemm_check_device_status(stream)
        med = statistics.median(per_step) * 1e-3
        ratio = FP8_OVER_BF16 if p.kind == "mxfp8" else 1.0
        measured = roofline_of(p.flops, min_bytes(p), med, float(peaks["bf16_tflops"]) * ratio,
                               float(peaks["hbm_gbs"]))
        nominal = roofline_of(p.flops, min_bytes(p), med, NOMINAL["bf16_tflops"] * ratio, NOMINAL["hbm_gbs"])
        entry = {"workload": p.desc, "M": p.M, "N": p.N, "K": p.K, "kernel_config": config_name(G, p, "auto"),
                 "launches_per_call": p.launches(G), "steps": steps,
                 "l2": ("flushed before every call (252 MiB written, then read back)" if flush else
                        "no flush (inputs+output > 2 x L2)"),
                 "median_us": med * 1e6, "p90_us": float(np.percentile(per_step, 90)) * 1e3,
                 # CUDA events on this GPU tick in 2.048 us steps, so a
                 # per-call median is a whole number of ticks; the mean of
                 # the calls resolves finer
                 "mean_us": statistics.fmean(per_step) * 1e3,
                 "tflops": p.flops / med / 1e12, "gbs": min_bytes(p) / med / 1e9,
                 "bound": measured["bound"], "roofline_us": measured["roofline_us"], "frac": measured["frac"],
                 "frac_of_nominal": nominal["frac"], "min_bytes": min_bytes(p)}
        if dirty:
            entry["median_us_after_dirty_flush"] = statistics.median(dirty) * 1e3
        if name == "single_tile128":
            # one 128 x 128 tile: launch latency, not a roofline, bounds it
            entry["bound"] = "latency"
            entry["graph_replay_us"] = graph_replay_us(p, G, dev, C, torch, stream, steps, scratch)
        out[name] = entry
        del dev, C
    del scratch
    return out


def config_name(G, p: Problem, forced: str) -> str:
    """Name of the kernel configuration a call of this problem runs."""
    if p.kind == "mxfp8":
        pair_tiles = ((p.M + 255) // 256) * ((p.N + 255) // 256)
        return forced if forced.startswith("mxfp8") else \
            ("mxfp8_2cta_256x256" if pair_tiles >= 74 else "mxfp8_1cta_128x256")
    name = {v: k for k, v in G.CONFIGS.items()}[G.gemm_select_config(p.M, p.N, p.K)]
    if p.kind == "fused" and forced == "auto" and name == "2cta_512x256_clc":
        name = "2cta_256x256_clc"   # the library's choice for a non-plain epilogue
    return name


def oracle_sample(problem: Problem, budget_s: float):
    """Time the CPU oracle on the first R rows of A (all of B), R sized so the
    run takes about budget_s.  Returns (flops, seconds, R)."""

    def timed(rows):
        t0 = time.perf_counter()
        problem.oracle_rows(rows)
        return time.perf_counter() - t0

    # each call decodes all of B once, then its threads share the rows of A:
    # time(r) ~ fixed + r * per_row once every thread has rows, so the two
    # calibration points are one and three rows per thread
    import oracle
    t = max(1, oracle.num_threads())
    t1, t3 = timed(min(problem.M, t)), timed(min(problem.M, 3 * t))
    per_row = max((t3 - t1) / (2.0 * t), 1e-6)
    fixed = max(t1 - t * per_row, 0.0)
    R = int(max(1, min(problem.M, (budget_s - fixed) / per_row)))
    if R > t:
        R -= R % t                          # whole rounds of rows per thread
    dt = timed(R)
    return 2.0 * R * problem.N * problem.K, dt, R


def needs_l2_flush(traffic_bytes: int) -> bool:
    """Inputs plus output under twice the L2 would be served partly from L2
    across back-to-back steps; those workloads flush it between steps."""
    return traffic_bytes < 2 * L2_BYTES


def metric_of(kind: str) -> str:
    return {"bf16": METRIC, "mxfp8": METRIC_MXFP8, "fused": METRIC_FUSED}[kind]


def run_reference(args, rank):
    """Reference arm: the CPU oracle, as it stands, on the host cores."""
    if rank != 0:
        return
    import oracle
    p = Problem(args.workload, args.shape, 0)
    # each step: a bounded row sample, sized so all warm-up + timed steps take
    # about two and a half minutes
    per_step = max(0.05, min(2.0, 150.0 / (args.steps + args.warmup)))
    _, _, R = oracle_sample(p, per_step)
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        p.oracle_rows(R)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = 2.0 * R * p.N * p.K * len(times) / total / 1e12
    line = {
        "impl": "reference", "metric": metric_of(p.kind), "value": value,
        "unit": UNIT, "n_gpus": 0, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": p.desc, "M": p.M, "N": p.N, "K": p.K, "sample_rows_per_step": R},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"rows 0..{R - 1} of A against all of B ({R}x{p.N}x{p.K}) per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


class _CublasCall:
    """cuBLAS (torch.mm) on a bf16 workload's device operands, called like Problem.call."""

    def __init__(self, torch):
        self.torch = torch

    def call(self, G, dev, C, stream):
        A, B = dev
        if C.dtype == self.torch.float32:
            self.torch.mm(A, B.t(), out_dtype=self.torch.float32, out=C)
        else:
            self.torch.mm(A, B.t(), out=C)


def cublas_context(args):
    """cuBLAS (torch.matmul / torch.mm) beside this library on one bf16 workload, in the
    same process and on the same stream, with bf16 and fp32 C for both: a 20-launch burst
    of each, then an args.steps-launch run of each, two interleaved rounds, back to back
    (no L2 flush: meant for shapes above 2 x L2, such as 8192^3).  Context for the reports,
    not a bench line: the JSON line says "context": "cublas", and the clock record covers
    the long runs.  The library path is the one `gemm_bf16` takes; cuBLAS is never on it."""
    import torch

    from dense_gemm_engineering_bf16_b200 import gemm as G

    p = Problem(args.workload, args.shape, 0)
    if p.kind != "bf16":
        raise SystemExit("--cublas-context: bf16 workloads only")
    A, B = p.device_arrays(torch)
    M, N, K = p.M, p.N, p.K
    C16 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    C32 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    Bt = B.t()                                   # K x N view of B stored N x K
    s = torch.cuda.current_stream()
    ops = {
        "cublas_bf16_out": lambda: torch.matmul(A, Bt, out=C16),
        "cublas_fp32_out": lambda: torch.mm(A, Bt, out_dtype=torch.float32, out=C32),
        "ours_bf16_out": lambda: G.gemm_bf16(A, B, C16, M, N, K, K, K, N, G.OUT_BF16, stream=s),
        "ours_fp32_out": lambda: G.gemm_bf16(A, B, C32, M, N, K, K, K, N, G.OUT_F32, stream=s),
    }

    def run(fn, steps):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(steps):
            fn()
        e1.record(s)
        torch.cuda.synchronize()
        return round(p.flops * steps / (e0.elapsed_time(e1) * 1e-3) / 1e12, 1)

    res = {name: {"burst_20": [], f"run_{args.steps}": []} for name in ops}
    for rnd in range(2):
        for name in (list(ops) if rnd == 0 else list(ops)[::-1]):
            res[name]["burst_20"].append(run(ops[name], 20))
    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
    except Exception:
        pass
    sampler = ClockSampler(gpu_id)
    sampler.start()
    for rnd in range(2):
        for name in (list(ops) if rnd == 0 else list(ops)[::-1]):
            res[name][f"run_{args.steps}"].append(run(ops[name], args.steps))
    sampler.stop()
    G.gemm_check_device_status(s)
    line = {"context": "cublas", "workload": p.desc, "unit": "TFLOP/s", "warmup": args.warmup, "results": res,
            "clocks": sampler.summary()}
    del A, B, C16, C32
    if args.configs and args.shape is None:
        # the bf16 workloads of the per-config report, each with the bench's
        # L2 rule: per call, median and mean (us) of args.config_steps calls,
        # three interleaved rounds
        scratch = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda")
        cub = _CublasCall(torch)
        per = {}
        for name in CONFIG_SET:
            q = Problem(name, None, 0)
            if q.kind != "bf16":
                continue
            dev = q.device_arrays(torch)
            C = q.empty_out(torch)
            flush = needs_l2_flush(min_bytes(q))
            r = {"ours": {"median_us": [], "mean_us": []}, "cublas": {"median_us": [], "mean_us": []}}
            for rnd in range(3):
                for tag, obj in ((("ours", q), ("cublas", cub)) if rnd % 2 == 0 else (("cublas", cub), ("ours", q))):
                    for _ in range(5):
                        obj.call(G, dev, C, s)
                    t, _ = time_steps(obj, G, dev, C, torch, s, args.config_steps, scratch if flush else None)
                    r[tag]["median_us"].append(round(statistics.median(t) * 1e3, 1))
                    r[tag]["mean_us"].append(round(statistics.fmean(t) * 1e3, 1))
            G.gemm_check_device_status(s)
            per[name] = {"shape": [q.M, q.N, q.K], "c": "fp32" if C.dtype == torch.float32 else "bf16",
                         "l2": "flushed before every call" if flush else "no flush", **r}
            del dev, C
        line["configs"] = per
    print(json.dumps(line))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="square8192", choices=sorted(WORKLOADS))
    ap.add_argument("--shape", type=int, nargs=3, metavar=("M", "N", "K"),
                    help="override the workload's shape (U[-1,1] inputs), e.g. for profiling")
    ap.add_argument("--config", default="auto")
    ap.add_argument("--e2e-steps", type=int, default=20, help="0 skips the end-to-end leg")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", dest="configs", action="store_false",
                    help="skip the per-config report (default run: every configuration's workload)")
    ap.add_argument("--config-steps", type=int, default=50)
    ap.add_argument("--cublas-context", action="store_true",
                    help="instead of the bench line: cuBLAS beside this library on the workload (context)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus > 1 and world == 1:
        raise SystemExit("--gpus N > 1 needs torchrun: python -m torch.distributed.run "
                         "--nproc-per-node N --master-addr 127.0.0.1 bench.py --gpus N")
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if args.cublas_context:
        if world > 1:
            raise SystemExit("--cublas-context runs on one GPU")
        cublas_context(args)
        return

    import torch
    import torch.distributed as dist

    from dense_gemm_engineering_bf16_b200 import gemm as G

    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    p = Problem(args.workload, args.shape, rank)
    dev = p.device_arrays(torch)
    C = p.empty_out(torch)
    G.gemm_force_config(args.config)
    cfg_name = config_name(G, p, args.config)
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        p.call(G, dev, C, stream)
    G.gemm_check_device_status(stream)

    # ---------------------------------------------------- timed region --
    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        pass
    # Working sets under twice the L2 would be served partly from L2 across
    # back-to-back steps: flush it between steps (write a buffer larger than
    # L2 outside the events) and time each step on its own.
    traffic_bytes = p.in_bytes + p.out_bytes
    flush = needs_l2_flush(traffic_bytes)
    scratch = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda") if flush else None
    sampler = ClockSampler(gpu_id)
    sampler.start()
    barrier()
    torch.cuda.synchronize()
    per_step_ms, span_ms = time_steps(p, G, dev, C, torch, stream, args.steps, scratch)
    barrier()
    sampler.stop()
    G.gemm_check_device_status(stream)
    local_ms = span_ms if span_ms is not None else sum(per_step_ms)
    t_ms = max_over_ranks(local_ms, world, "cuda")

    fusion = fusion_comparison(p, G, dev, torch, stream, min(args.steps, 50)) if p.kind == "fused" else None

    # ------------------------------------------- end to end, host buffers --
    # Every step copies its inputs from pinned host memory, runs the call and
    # copies its result back.  The steps are pipelined the way a caller
    # streaming batches would run them: inputs go up on one copy stream,
    # results come down on another, and the GEMM runs on the compute stream,
    # with two sets of device buffers so that step i + 1's upload and step
    # i - 1's download overlap step i's GEMM (PCIe is full duplex).  The
    # serial form (one stream, copy - call - copy) is reported beside it.
    e2e = None
    if args.e2e_steps > 0:
        host = [torch.from_numpy(np.ascontiguousarray(x).view(np.int16 if x.dtype == np.uint16 else np.uint8))
                .pin_memory() for x in p.host]
        dev_e = [[torch.empty_like(d) for d in dev] for _ in range(2)]
        C_h = [p.empty_out(torch, pinned=True) for _ in range(2)]
        C_e = [p.empty_out(torch) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()  # noqa: E731
        up_done = [ev(), ev()]           # inputs of buffer b uploaded
        gemm_done = [ev(), ev()]         # GEMM into buffer b finished (its inputs are free)
        down_done = [ev(), ev()]         # result of buffer b downloaded (its C is free)

        def upload(b):
            with torch.cuda.stream(s_in):
                for d, h in zip(dev_e[b], host):
                    d.view(h.dtype).copy_(h, non_blocking=True)
            up_done[b].record(s_in)

        def pipelined(steps, start):
            s_in.wait_event(start)
            for b in range(min(2, steps)):
                upload(b)
            for i in range(steps):
                b = i % 2
                stream.wait_event(up_done[b])
                stream.wait_event(down_done[b])
                p.call(G, dev_e[b], C_e[b], stream)
                gemm_done[b].record(stream)
                s_out.wait_event(gemm_done[b])
                with torch.cuda.stream(s_out):
                    C_h[b].copy_(C_e[b], non_blocking=True)
                down_done[b].record(s_out)
                if i + 2 < steps:
                    s_in.wait_event(gemm_done[b])
                    upload(b)
            stream.wait_stream(s_out)

        def serial_step():
            for d, h in zip(dev_e[0], host):
                d.view(h.dtype).copy_(h, non_blocking=True)
            p.call(G, dev_e[0], C_e[0], stream)
            C_h[0].copy_(C_e[0], non_blocking=True)

        warm = torch.cuda.Event()
        warm.record(stream)
        pipelined(2, warm)
        serial_step()
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        pipelined(args.e2e_steps, e0)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, "cuda")
        barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.e2e_steps):
            serial_step()
        f1.record(stream)
        torch.cuda.synchronize()
        serial_ms = max_over_ranks(f0.elapsed_time(f1), world, "cuda")
        barrier()
        G.gemm_check_device_status(stream)
        e2e = {"value": whole_job_tflops(p.flops, args.e2e_steps, world, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": p.in_bytes, "d2h_bytes_per_step": p.out_bytes, "steps": args.e2e_steps,
               "pipeline": "inputs up on one copy stream, results down on another, GEMM on the compute stream; "
                           "two buffer sets",
               "serial_value": whole_job_tflops(p.flops, args.e2e_steps, world, serial_ms)}

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_src = load_peaks()
    for key, v in FALLBACK_PEAKS.items():
        peaks.setdefault(key, v)
    configs = None
    if args.configs and world == 1 and args.shape is None and args.workload == "square8192":
        G.gemm_force_config("auto")
        csampler = ClockSampler(gpu_id)
        csampler.start()
        configs = config_report(G, torch, stream, peaks, args.config_steps, 5)
        csampler.stop()
        configs["clocks"] = csampler.summary()
        G.gemm_force_config(args.config)

    value = whole_job_tflops(p.flops, args.steps, world, t_ms)
    # per-step event time: for bf16 the step is the one GEMM launch; for
    # MXFP8 it also holds the small scale-repack launch, so `achieved` is a
    # lower bound for the GEMM kernel alone
    mean_step_s = sum(per_step_ms) / len(per_step_ms) * 1e-3
    bf16_peak = float(peaks["bf16_tflops"])
    sustained = float(peaks["bf16_tflops_sustained"])
    ratio = FP8_OVER_BF16 if p.kind == "mxfp8" else 1.0
    roofline = roofline_of(p.flops, min_bytes(p), mean_step_s, bf16_peak * ratio, float(peaks["hbm_gbs"]))
    nominal = roofline_of(p.flops, min_bytes(p), mean_step_s, NOMINAL["bf16_tflops"] * ratio, NOMINAL["hbm_gbs"])
    if roofline["bound"] == "tensor":
        peak_note = (f"{peak_src} bf16_tflops (burst, cuBLAS 8192^3)" if p.kind != "mxfp8" else
                     f"{peak_src} bf16_tflops x {FP8_OVER_BF16:g} (nominal fp8/bf16 dense ratio)")
    else:
        peak_note = f"{peak_src} hbm_gbs (copy bandwidth)"
    roofline.update({
        "traffic": profile_traffic(p.name, cfg_name), "peak_source": peak_note,
        "frac_of_nominal_peak": nominal["frac"],
        "nominal_peak": nominal["peak"],
        "frac_of_sustained_peak": (p.flops / mean_step_s / 1e12) / (sustained * ratio),
        "algorithmic_flops_per_launch": p.flops,
        "min_bytes_per_launch": min_bytes(p)})

    cpu = None
    if not args.no_cpu_baseline:
        import oracle
        fl, dt, R = oracle_sample(p, args.cpu_budget)
        cpu = {"value": fl / dt / 1e12, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
               "sample": f"rows 0..{R - 1} of A against all of B ({R}x{p.N}x{p.K}), fp64 triple loop, "
                         f"{dt:.1f} s"}

    line = {
        "metric": metric_of(p.kind), "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3" if p.kind == "mxfp8" else "bf16",
        "data": "synthetic",
        "config": {"workload": p.desc, "M": p.M, "N": p.N, "K": p.K, "kernel_config": cfg_name,
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": (f"flushed between steps ({2 * L2_BYTES // 2**20} MiB written, then read back, outside "
                          f"the events): "
                          f"inputs+output {traffic_bytes / 2**20:.0f} MiB < 2 x 126 MiB L2" if flush else
                          f"no flush: inputs+output {traffic_bytes / 2**20:.0f} MiB > 2 x 126 MiB L2"),
                   "step_ms_median": statistics.median(per_step_ms),
                   "step_ms_p90": float(np.percentile(per_step_ms, 90))},
        "e2e": e2e,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "clocks": sampler.summary(),
        "gpu_launches": args.steps * p.launches(G) * world,
    }
    if configs:
        line["configs"] = configs
    if fusion:
        hbm = float(peaks["hbm_gbs"])
        fusion["ledger_saved_ms_at_hbm_peak"] = fusion["ledger_saved_bytes"] / (hbm * 1e9) * 1e3
        fusion["unfused_pass_frac_of_hbm_peak"] = fusion["unfused_pass_gbs"] / hbm
        line["fusion"] = fusion
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
