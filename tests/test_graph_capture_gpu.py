"""CUDA-graph capture of the GEMM calls: fixed shapes, reusable addresses,
one-time set-up kept out of the capture, and replays that stay correct
after a workspace grows ("GPU 执行模型", section "Launch、CUDA Graph 与动态
shape").  The fresh-process cases run tests/graph_capture_child.py."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
from dense_gemm_engineering_bf16_b200 import gemm as G
from dense_gemm_engineering_bf16_b200 import synth

from gpu_helpers import to_device_bf16

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def _child(case):
    out = subprocess.run([sys.executable, os.path.join(HERE, "graph_capture_child.py"), case],
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-3000:]
    return json.loads(out.stdout.strip().splitlines()[-1])


def test_set_up_is_refused_inside_capture_then_replays_are_correct():
    r = _child("refuse_then_replay")
    assert r["first_call_in_capture"] == 8, r          # GEMM_ERR_CAPTURE, nothing queued
    assert r["c_untouched"], r
    assert r["warm_up"] == 0 and r["capture_after_warm_up"] == 0, r
    assert r["replay_max_excess"] <= 0.0, r
    assert r["status"] == 0, r


def test_replays_stay_valid_after_the_workspaces_grow():
    r = _child("growth_after_capture")
    assert r["skinny_selected"], r
    assert r["skinny_warm_up"] == 0 and r["skinny_capture"] == 0, r
    assert r["big_skinny_in_capture"] == 8 and r["big_skinny"] == 0, r
    assert r["skinny_replay_max_excess"] <= 0.0, r
    assert r["mx_warm_up"] == 0 and r["mx_capture"] == 0 and r["big_mx"] == 0, r
    assert r["mx_replay_max_excess"] <= 0.0, r
    assert r["status"] == 0, r


def test_one_graph_of_several_configs_replays_like_eager_calls():
    """One graph holding the 2-CTA CLC kernel (4096 x 4096), the skinny path
    (32 rows), the fused epilogue (bias + ReLU, bf16 out) and the
    block-scaled path; replayed with fresh inputs, every output is
    bit-identical to the same calls made eagerly."""
    s = torch.cuda.Stream()
    M1, N1, K1 = 4096, 4096, 2560
    a1, b1 = synth.bf16_operands(M1, N1, K1, "uniform", workload=420)
    A1, B1 = to_device_bf16(a1), to_device_bf16(b1)
    C1 = torch.empty((M1, N1), dtype=torch.float32, device="cuda")
    M2, N2, K2 = 32, 2048, 8192
    a2, b2 = synth.bf16_operands(M2, N2, K2, "normal", workload=421)
    A2, B2 = to_device_bf16(a2), to_device_bf16(b2)
    C2 = torch.empty((M2, N2), dtype=torch.float32, device="cuda")
    M3, N3, K3 = 300, 520, 1024
    a3, b3 = synth.bf16_operands(M3, N3, K3, "normal", workload=422)
    A3, B3 = to_device_bf16(a3), to_device_bf16(b3)
    bias = torch.from_numpy(synth.normal(423, (N3,)).astype(np.float32)).cuda()
    C3 = torch.empty((M3, N3), dtype=torch.bfloat16, device="cuda")
    M4 = N4 = K4 = 512
    am, sa, bm, sb = synth.mxfp8_operands(M4, N4, K4, workload=424)
    A4, B4 = torch.from_numpy(am).cuda(), torch.from_numpy(bm).cuda()
    SA, SB = torch.from_numpy(sa).cuda(), torch.from_numpy(sb).cuda()
    C4 = torch.empty((M4, N4), dtype=torch.bfloat16, device="cuda")
    assert G.gemm_select_config(M1, N1, K1) == G.CONFIGS["2cta_256x256_clc"]
    assert G.gemm_select_config(M2, N2, K2) == G.CONFIGS["skinny"]

    def calls():
        G.gemm_bf16(A1, B1, C1, M1, N1, K1, K1, K1, N1, stream=s)
        G.gemm_bf16(A2, B2, C2, M2, N2, K2, K2, K2, N2, stream=s)
        G.gemm_bf16_fused(A3, B3, C3, M3, N3, K3, K3, K3, N3, G.OUT_BF16, G.KMAJOR, G.KMAJOR, 1.0, 0.0,
                          bias, G.ACT_RELU, stream=s)
        G.gemm_mxfp8(A4, SA, B4, SB, C4, M4, N4, K4, K4, K4, N4, stream=s)

    with torch.cuda.stream(s):
        calls()                                   # warm-up: set-up happens here
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        calls()
    for rep in range(2):
        for t in (A1, B1, A2, B2, A3, B3):
            t.copy_(torch.randn(t.shape, device="cuda").to(torch.bfloat16))
        for t in (C1, C2, C3, C4):
            t.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        got = [t.clone() for t in (C1, C2, C3, C4)]
        with torch.cuda.stream(s):
            calls()
        s.synchronize()
        for x, y in zip(got, (C1, C2, C3, C4)):
            assert torch.equal(x, y)
    # the last replay's fused output against the oracle, on sampled rows
    a3_bits = A3.view(torch.int16).cpu().numpy().view(np.uint16)
    b3_bits = B3.view(torch.int16).cpu().numpy().view(np.uint16)
    rows = np.arange(0, M3, 7)
    c_ab, s_abs = oracle.gemm_bf16_f64(a3_bits, b3_bits, rows=rows, with_abs=True)
    want = oracle.epilogue(c_ab, None, 1.0, 0.0, bias.cpu().numpy().astype(np.float64), oracle.ACT_RELU)
    tol = 1e-3 * s_abs + 1e-6 + 2.0 ** -8 * np.abs(want)
    assert np.all(np.abs(C3.cpu().float().numpy()[rows] - want) <= tol)
    assert G.gemm_check_device_status() == 0


def test_stream_k_replays_match_eager_and_oracle():
    """The stream-K kernel in a graph: its split-tile counters are left at
    zero arrivals by each launch, so replays (same epoch) stay correct."""
    s = torch.cuda.Stream()
    M, N, K = 1000, 1500, 1000                 # 4 x 6 = 24 pair tiles x 16 K blocks over <= 74 pairs
    a, b = synth.bf16_operands(M, N, K, "normal", workload=430)
    A, B = to_device_bf16(a), to_device_bf16(b)
    C = torch.empty((M, N), dtype=torch.float32, device="cuda")
    G.gemm_force_config("2cta_256x256_sk")
    try:
        call = lambda: G.gemm_bf16(A, B, C, M, N, K, K, K, N, stream=s)  # noqa: E731
        with torch.cuda.stream(s):
            call()
        s.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            call()
        for rep in range(3):
            a2, b2 = synth.bf16_operands(M, N, K, "normal", workload=431 + rep)
            A.copy_(to_device_bf16(a2))
            B.copy_(to_device_bf16(b2))
            C.fill_(float("nan"))
            g.replay()
            torch.cuda.synchronize()
            got = C.clone()
            with torch.cuda.stream(s):
                call()
            s.synchronize()
            assert torch.equal(got, C)
            rows = np.arange(0, M, 37)
            c_ref, s_abs = oracle.gemm_bf16_f64(a2, b2, rows=rows, with_abs=True)
            err = np.abs(got.cpu().numpy()[rows].astype(np.float64) - c_ref)
            assert np.all(err <= 1e-3 * s_abs + 1e-6)
    finally:
        G.gemm_force_config("auto")
    G.gemm_check_device_status()


def test_cluster_split_k_replays_match_eager_and_oracle():
    """The cluster split-K kernel in a graph: its cluster barriers start each
    launch afresh, so replays with new inputs give the eager bits."""
    s = torch.cuda.Stream()
    M, N, K = 256, 2048, 4096                  # 32 tiles of 128 x 128: clusters of four over K
    assert G.gemm_select_config(M, N, K) == G.CONFIGS["1cta_128x128_splitk"]
    a, b = synth.bf16_operands(M, N, K, "normal", workload=440)
    A, B = to_device_bf16(a), to_device_bf16(b)
    C = torch.empty((M, N), dtype=torch.float32, device="cuda")
    call = lambda: G.gemm_bf16(A, B, C, M, N, K, K, K, N, stream=s)  # noqa: E731
    with torch.cuda.stream(s):
        call()
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        call()
    for rep in range(3):
        a2, b2 = synth.bf16_operands(M, N, K, "normal", workload=441 + rep)
        A.copy_(to_device_bf16(a2))
        B.copy_(to_device_bf16(b2))
        C.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        got = C.clone()
        with torch.cuda.stream(s):
            call()
        s.synchronize()
        assert torch.equal(got, C)
    rows = np.arange(0, M, 5)
    c_ref, s_abs = oracle.gemm_bf16_f64(a2, b2, rows=rows, with_abs=True)
    assert np.all(np.abs(C.cpu().numpy()[rows].astype(np.float64) - c_ref) <= 1e-3 * s_abs + 1e-6)
    del g
    assert G.gemm_check_device_status() == 0
