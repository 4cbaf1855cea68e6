"""Benchmark: bf16 GEMM TFLOP/s at 8192^3 on B200 (C = A.B, bf16 in, fp32 accumulate and out).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload square8192|square4096|ragged|skinny1000|skinny16]

One step = one gemm_bf16 call over the whole M x N x K problem, inputs
resident in HBM.  Multi-GPU runs (torchrun, one process per GPU) are
independent replicas: every rank multiplies its own seeded matrices, no data
crosses GPUs, and value = FLOPs of all ranks / the slowest rank's time.

Printed (rank 0): one JSON line with the metric, the device-timed value,
`e2e` (same metric through the C ABI with host buffers, copies included),
`roofline` of the GEMM kernel, `cpu_baseline` (the CPU oracle on a bounded
sample of the same workload), clocks sampled during the timed region and the
number of kernel launches.  `--impl reference` times the oracle alone as the
reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import glob
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "bf16 GEMM TFLOP/s at 8192³ on 1 B200 (fraction of dense BF16 tensor peak)"
UNIT = "TFLOP/s"

WORKLOADS = {
    # name: (M, N, K, distribution, workload id, description)
    "square8192": (8192, 8192, 8192, "uniform", 3, "gemm 8192x8192x8192, bf16 U[-1,1] in, fp32 accumulate + out"),
    "square4096": (4096, 4096, 4096, "normal_scaled", 2, "gemm 4096x4096x4096, bf16 N(0,1)/sqrt(K) in, fp32 out"),
    "ragged": (4000, 3000, 2000, "normal", 4, "gemm 4000x3000x2000, bf16 N(0,1) in, fp32 out"),
    "skinny1000": (1000, 8192, 8192, "normal", 5, "gemm 1000x8192x8192, bf16 N(0,1) in, fp32 out"),
    "skinny16": (16, 8192, 8192, "normal", 6, "gemm 16x8192x8192, bf16 N(0,1) in, fp32 out"),
}

L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for p in sorted(glob.glob(os.path.join(ROOT, "dense_gemm_engineering_bf16_b200", "csrc", "*"))):
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def profile_traffic(workload: str, config_name: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    entry = t.get(f"{workload}:{config_name}")
    if not entry or entry.get("kernel_source_hash") != kernel_source_hash():
        return None
    return entry.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle samples every 100 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
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
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus > 1 and world == 1:
        raise SystemExit("--gpus N > 1 needs torchrun: python -m torch.distributed.run "
                         "--nproc-per-node N --master-addr 127.0.0.1 bench.py --gpus N")
    return world, rank, local


def oracle_sample(a_bits, b_bits, K, budget_s):
    """Time the CPU oracle on the first R rows of A (all of B), R sized so
    the run takes about budget_s.  Returns (flops, seconds, R)."""
    import oracle

    def timed(rows):
        t0 = time.perf_counter()
        oracle.gemm_bf16_f64(a_bits[:rows], b_bits, K=K)
        return time.perf_counter() - t0

    # each call decodes all of B once, then spends a fixed time per row of A:
    # two calibration points give both parts
    t4, t16 = timed(4), timed(16)
    per_row = max((t16 - t4) / 12.0, 1e-6)
    fixed = max(t4 - 4 * per_row, 0.0)
    R = int(max(4, min(a_bits.shape[0], (budget_s - fixed) / per_row)))
    t0 = time.perf_counter()
    oracle.gemm_bf16_f64(a_bits[:R], b_bits, K=K)
    dt = time.perf_counter() - t0
    return 2.0 * R * b_bits.shape[0] * K, dt, R


def run_reference(args, world, rank):
    """Reference arm: the CPU oracle, as it stands, on the host cores."""
    if rank != 0:
        return
    import oracle
    from dense_gemm_engineering_bf16_b200 import synth
    M, N, K, dist, wid, desc = WORKLOADS[args.workload]
    a_bits, b_bits = synth.bf16_operands(M, N, K, dist, workload=wid)
    # each step: a bounded row sample of the workload, sized so that all
    # warm-up + timed steps take about two and a half minutes
    per_step = max(0.05, min(2.0, 150.0 / (args.steps + args.warmup)))
    _, _, R = oracle_sample(a_bits, b_bits, K, budget_s=per_step)
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle.gemm_bf16_f64(a_bits[:R], b_bits, K=K)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = 2.0 * R * N * K * len(times) / total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 0,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": desc, "M": M, "N": N, "K": K,
                                        "sample_rows_per_step": R},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"rows 0..{R - 1} of A against all of B ({R}x{N}x{K}) per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="square8192", choices=sorted(WORKLOADS))
    ap.add_argument("--shape", type=int, nargs=3, metavar=("M", "N", "K"),
                    help="override the workload's shape (bf16 U[-1,1] inputs), e.g. for profiling")
    ap.add_argument("--config", default="auto")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        run_reference(args, world, rank)
        return

    import torch
    import torch.distributed as dist

    from dense_gemm_engineering_bf16_b200 import gemm as G
    from dense_gemm_engineering_bf16_b200 import synth

    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    M, N, K, distname, wid, desc = WORKLOADS[args.workload]
    if args.shape:
        M, N, K = args.shape
        distname, wid = "uniform", 90
        desc = f"gemm {M}x{N}x{K}, bf16 U[-1,1] in, fp32 out"
    a_bits, b_bits = synth.bf16_operands(M, N, K, distname, workload=wid, base=rank)
    A = torch.from_numpy(a_bits.view(np.int16)).cuda().view(torch.bfloat16)
    B = torch.from_numpy(b_bits.view(np.int16)).cuda().view(torch.bfloat16)
    C = torch.empty((M, N), dtype=torch.float32, device="cuda")
    G.gemm_force_config(args.config)
    cfg_id = G.gemm_select_config(M, N, K)
    cfg_name = {v: k for k, v in G.CONFIGS.items()}[cfg_id]
    stream = torch.cuda.current_stream()
    flops = 2.0 * M * N * K
    in_out_bytes = 2 * (M * K + N * K) + 4 * M * N

    def step():
        G.gemm_bf16(A, B, C, M, N, K, K, K, N, G.OUT_F32, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    G.gemm_check_device_status(stream)

    # ---------------------------------------------------- timed region --
    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        pass
    sampler = ClockSampler(gpu_id)
    sampler.start()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    barrier()
    torch.cuda.synchronize()
    ev[0].record(stream)
    for i in range(args.steps):
        step()
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    barrier()
    sampler.stop()
    G.gemm_check_device_status(stream)
    per_launch_ms = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    t_ms = ev[0].elapsed_time(ev[-1])
    if world > 1:
        t = torch.tensor([t_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        t_ms = float(t.item())
    # ------------------------------------------- end to end, host buffers --
    e2e_steps = args.e2e_steps
    e2e_value = None
    if e2e_steps > 0:
        e2e_value = run_e2e(torch, dist, G, a_bits, b_bits, A, B, C, M, N, K, flops, e2e_steps,
                            stream, world, barrier)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    _report(args, G, M, N, K, desc, cfg_name, flops, in_out_bytes, world, t_ms, per_launch_ms,
            sampler, e2e_value, e2e_steps, a_bits, b_bits)


def run_e2e(torch, dist, G, a_bits, b_bits, A, B, C, M, N, K, flops, e2e_steps, stream, world, barrier):
    """Same metric through the C ABI with pinned host buffers: H2D of A and B,
    the GEMM, D2H of C, all inside the timed region."""
    A_h = torch.from_numpy(a_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    B_h = torch.from_numpy(b_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    C_h = torch.empty((M, N), dtype=torch.float32).pin_memory()
    A_d = torch.empty_like(A)
    B_d = torch.empty_like(B)
    C_d = torch.empty_like(C)

    def e2e_step():
        A_d.copy_(A_h, non_blocking=True)
        B_d.copy_(B_h, non_blocking=True)
        G.gemm_bf16(A_d, B_d, C_d, M, N, K, K, K, N, G.OUT_F32, stream=stream)
        C_h.copy_(C_d, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    if world > 1:
        t = torch.tensor([e2e_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    barrier()
    G.gemm_check_device_status(stream)
    return world * e2e_steps * flops / (e2e_ms * 1e-3) / 1e12


def _report(args, G, M, N, K, desc, cfg_name, flops, in_out_bytes, world, t_ms, per_launch_ms,
            sampler, e2e_value, e2e_steps, a_bits, b_bits):
    value = world * args.steps * flops / (t_ms * 1e-3) / 1e12
    # ------------------------------------------------------------ roofline --
    peaks, peak_src = load_peaks()
    mean_launch_ms = sum(per_launch_ms) / len(per_launch_ms)
    achieved = flops / (mean_launch_ms * 1e-3) / 1e12
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    traffic = profile_traffic(args.workload, cfg_name)
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic,
                "peak_source": f"{peak_src} bf16_tflops (burst, cuBLAS 8192^3)",
                "algorithmic_flops_per_launch": flops,
                "min_bytes_per_launch": in_out_bytes}

    cpu = None
    if not args.no_cpu_baseline:
        import oracle
        fl, dt, R = oracle_sample(a_bits, b_bits, K, budget_s=args.cpu_budget)
        cpu = {"value": fl / dt / 1e12, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
               "sample": f"rows 0..{R - 1} of A against all of B ({R}x{N}x{K}), fp64 triple loop, "
                         f"{dt:.1f} s"}

    clocks = sampler.summary()
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": desc, "M": M, "N": N, "K": K, "kernel_config": cfg_name,
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": f"no flush: inputs+output {in_out_bytes / 2**20:.0f} MiB > 126 MiB L2"
                   if in_out_bytes > L2_BYTES else "inputs fit in L2 (not flushed)",
                   "launch_ms_median": statistics.median(per_launch_ms),
                   "launch_ms_p90": float(np.percentile(per_launch_ms, 90))},
        "e2e": None if e2e_value is None else
        {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": 2 * (M * K + N * K),
         "d2h_bytes_per_step": 4 * M * N, "steps": e2e_steps},
        "roofline": roofline,
        "cpu_baseline": cpu,
        "clocks": clocks,
        "gpu_launches": args.steps * G.gemm_launches_per_call(M, N, K, False) * world,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
