"""Host-side logic of bench.py on CPU: the multi-rank (replicas) timing rule
on two gloo ranks, the clock-sample summary, the oracle sample sizing and the
reference arm's rank handling.  No GPU."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # every rank ran 10 steps of 1 TFLOP; rank 1 was slower
        local_ms = 100.0 if rank == 0 else 250.0
        slowest = bench.max_over_ranks(local_ms, world, "cpu")
        value = bench.whole_job_tflops(1e12, 10, world, slowest)
        q.put((rank, slowest, value))
    finally:
        dist.destroy_process_group()


def test_replicas_take_the_slowest_rank_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, slowest, value in got:
        assert slowest == 250.0
        assert value == pytest.approx(2 * 10 * 1e12 / 0.25 / 1e12)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_tflops(2e12, 4, 1, 8.0) == pytest.approx(1000.0)


def test_clock_summary_reads_reasons_and_median():
    lines = [
        "0, 1965, 1965, 950.1, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1800, 1965, 999.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1500, 1965, 990.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]
    s = bench.summarize_clocks(lines)
    assert s["sm_mhz"] == 1800 and s["sm_max_mhz"] == 1965 and s["samples"] == 3
    assert s["samples_under_load"] == 3
    assert s["reasons"] == ["sw_power_cap"]
    assert bench.summarize_clocks([])["samples"] == 0
    idle_then_busy = ["0, 1965, 1965, 200.0, 0x0, Not Active, Not Active, Not Active, Not Active"] * 5 + \
        ["0, 1400, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active"] * 3
    s = bench.summarize_clocks(idle_then_busy)
    assert s["sm_mhz"] == 1400 and s["samples_under_load"] == 3


def test_workloads_match_the_named_configs():
    assert bench.WORKLOADS["square8192"][:4] == (8192, 8192, 8192, "bf16")
    assert bench.WORKLOADS["skinny16"][:3] == (16, 8192, 8192)
    assert bench.WORKLOADS["mxfp8_8192"][3] == "mxfp8"


def test_oracle_sample_is_bounded():
    p = bench.Problem("square4096", (64, 96, 128), 0)
    flops, dt, rows = bench.oracle_sample(p, budget_s=0.05)
    assert 1 <= rows <= 64 and flops == 2.0 * rows * 96 * 128 and dt < 5


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--gpus", "2", "--steps", "1", "--warmup", "3"],
                         env=env, capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_reference_arm_prints_one_line_on_rank0():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--shape", "64", "128", "256", "--steps", "2", "--warmup", "3"],
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_kernel_hash_ignores_comments_only():
    import bench
    a = "int f() { return 1; }  // one\n/* block\n comment */\nint g;\n"
    b = "// header\nint f() { return 1; }\n\n\nint g;   /* trailing */\n"
    c = "int f() { return 2; }\nint g;\n"
    assert bench.code_only(a) == bench.code_only(b)
    assert bench.code_only(a) != bench.code_only(c)
    for kernel in bench.KERNEL_SOURCES:
        assert len(bench.kernel_source_hash(kernel)) == 16


def test_only_the_8192_cubes_run_without_an_l2_flush():
    for name in bench.WORKLOADS:
        p = bench.Problem(name, (8, 8, 32), 0)          # the byte counts below use the full sizes
        M, N, K, kind = bench.WORKLOADS[name][:4]
        in_b = {"bf16": 2 * (M * K + N * K), "fused": 2 * (M * K + N * K) + 4 * N,
                "mxfp8": M * K + N * K + (M + N) * (K // 32)}[kind]
        out_b = 4 * M * N if kind == "bf16" else 2 * M * N
        assert bench.needs_l2_flush(in_b + out_b) == (M != 8192), name
        assert p.kind == kind


def test_fused_workloads_use_their_activation_in_the_oracle_leg():
    import numpy as np
    import oracle
    for name, act in (("fused8192", oracle.ACT_GELU), ("fused8192_tanh", oracle.ACT_GELU_TANH)):
        p = bench.Problem(name, (4, 8, 64), 0)
        got = p.oracle_rows(4)
        base = oracle.gemm_bf16_f64(p.a[:4], p.b, K=64)
        want = oracle.epilogue(base, None, 1.0, 0.0, p.bias.astype(np.float64), act)
        assert np.array_equal(got, want)
    assert bench.metric_of("fused") == bench.METRIC_FUSED and bench.metric_of("mxfp8") == bench.METRIC_MXFP8


def test_roofline_takes_the_larger_of_compute_and_bandwidth():
    # 8192^3: 1.1e12 FLOP over 1686 TFLOP/s (652 us) outweighs 537 MB over 6549 GB/s (82 us)
    r = bench.roofline_of(2.0 * 8192 ** 3, 536870912, 0.72e-3, 1686.0, 6549.0)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["frac"] - (2.0 * 8192 ** 3 / 1686e12) / 0.72e-3) < 1e-12
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-12
    # 16 x 8192 x 8192: 2.1 GFLOP (1.3 us) against 135 MB (20.6 us): HBM-bound
    nbytes = 2 * (16 * 8192 + 8192 * 8192) + 4 * 16 * 8192
    r = bench.roofline_of(2.0 * 16 * 8192 * 8192, nbytes, 40e-6, 1686.0, 6549.0)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-12
    assert 0.5 < r["frac"] < 0.53


def test_config_set_covers_every_named_configuration():
    shapes = {bench.WORKLOADS[n][:3] for n in bench.CONFIG_SET} | {bench.WORKLOADS["square8192"][:3]}
    for want in [(128, 128, 128), (4096, 4096, 4096), (8192, 8192, 8192), (4000, 3000, 2000),
                 (1000, 8192, 8192), (16, 8192, 8192)]:
        assert want in shapes
    assert bench.WORKLOADS["mxfp8_8192"][3] == "mxfp8" and "mxfp8_8192" in bench.CONFIG_SET
    p = bench.Problem("square4096_bf16", (8, 8, 32), 0)
    assert p.bf16_out and p.out_bytes == 2 * 8 * 8


def test_cublas_context_mode_refuses_what_it_cannot_compare():
    """`--cublas-context` prints context, not a bench line: it runs on one GPU
    and only on bf16 workloads (the block-scaled one has no torch.mm twin),
    and it says so before touching a device."""
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--cublas-context", "--workload",
                          "mxfp8_8192"], capture_output=True, text=True, timeout=300)
    assert out.returncode != 0 and "bf16 workloads only" in out.stderr
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--cublas-context"], capture_output=True,
                         text=True, timeout=300, env=env)
    assert out.returncode != 0 and "one GPU" in out.stderr
