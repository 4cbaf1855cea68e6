"""Run in a fresh process by test_graph_capture_gpu.py (a fresh process has
no device state, kernel attributes or workspaces yet).  Prints one JSON
line with what it saw; the parent asserts on it."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import numpy as np  # noqa: E402
import torch  # noqa: E402

import oracle  # noqa: E402
from dense_gemm_engineering_bf16_b200 import gemm as G  # noqa: E402
from dense_gemm_engineering_bf16_b200 import synth  # noqa: E402


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def max_excess(got, c_ref, s_abs):
    return float(np.max(np.abs(got - c_ref) - (1e-3 * s_abs + 1e-6)))


def capture(fn, stream):
    g = torch.cuda.CUDAGraph()
    out = {}
    with torch.cuda.graph(g, stream=stream):
        out["status"] = fn()
    return g, out["status"]


def refuse_then_replay():
    res = {}
    M = N = K = 512
    a_bits, b_bits = synth.bf16_operands(M, N, K, "uniform", workload=400)
    A, B = dev_bf16(a_bits), dev_bf16(b_bits)
    C = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    call = lambda: G.gemm_bf16(A, B, C, M, N, K, K, K, N, stream=s, check=False)  # noqa: E731
    _, res["first_call_in_capture"] = capture(call, s)
    res["c_untouched"] = bool((C == 0).all().item())
    with torch.cuda.stream(s):
        res["warm_up"] = call()
    s.synchronize()
    g, res["capture_after_warm_up"] = capture(call, s)
    excess = []
    for rep in range(3):
        a2, b2 = synth.bf16_operands(M, N, K, "uniform", workload=401 + rep)
        A.copy_(dev_bf16(a2))
        B.copy_(dev_bf16(b2))
        C.zero_()
        g.replay()
        torch.cuda.synchronize()
        c_ref, s_abs = oracle.gemm_bf16_f64(a2, b2, with_abs=True)
        excess.append(max_excess(C.cpu().numpy().astype(np.float64), c_ref, s_abs))
    res["replay_max_excess"] = max(excess)
    res["status"] = G.gemm_check_device_status(check=False)
    return res


def growth_after_capture():
    res = {}
    s = torch.cuda.Stream()
    # skinny: small problem captured, then a large one grows the workspace
    m, n, k = 16, 256, 8192
    a_bits, b_bits = synth.bf16_operands(m, n, k, "normal", workload=410)
    A, B = dev_bf16(a_bits), dev_bf16(b_bits)
    C = torch.zeros((m, n), dtype=torch.float32, device="cuda")
    call = lambda: G.gemm_bf16(A, B, C, m, n, k, k, k, n, stream=s, check=False)  # noqa: E731
    res["skinny_selected"] = G.gemm_select_config(m, n, k) == G.CONFIGS["skinny"]
    with torch.cuda.stream(s):
        res["skinny_warm_up"] = call()
    s.synchronize()
    g_sk, res["skinny_capture"] = capture(call, s)
    big_m, big_n, big_k = 32, 2048, 8192       # 16 tiles of B: stream-K, a larger workspace
    A2 = torch.zeros((big_m, big_k), dtype=torch.bfloat16, device="cuda")
    B2 = torch.zeros((big_n, big_k), dtype=torch.bfloat16, device="cuda")
    C2 = torch.empty((big_m, big_n), dtype=torch.float32, device="cuda")
    res["big_skinny_in_capture"] = capture(
        lambda: G.gemm_bf16(A2, B2, C2, big_m, big_n, big_k, big_k, big_k, big_n, stream=s, check=False), s)[1]
    res["big_skinny"] = G.gemm_bf16(A2, B2, C2, big_m, big_n, big_k, big_k, big_k, big_n, check=False)
    torch.cuda.synchronize()
    a3, b3 = synth.bf16_operands(m, n, k, "normal", workload=411)
    A.copy_(dev_bf16(a3))
    B.copy_(dev_bf16(b3))
    g_sk.replay()
    torch.cuda.synchronize()
    c_ref, s_abs = oracle.gemm_bf16_f64(a3, b3, with_abs=True)
    res["skinny_replay_max_excess"] = max_excess(C.cpu().numpy().astype(np.float64), c_ref, s_abs)

    # block-scaled: the same with the repacked-scale workspace
    m = n = k = 256
    a_c, sfa, b_c, sfb = synth.mxfp8_operands(m, n, k, workload=412)
    dA, dB = torch.from_numpy(a_c).cuda(), torch.from_numpy(b_c).cuda()
    dsa, dsb = torch.from_numpy(sfa).cuda(), torch.from_numpy(sfb).cuda()
    Cm = torch.zeros((m, n), dtype=torch.bfloat16, device="cuda")
    mcall = lambda: G.gemm_mxfp8(dA, dsa, dB, dsb, Cm, m, n, k, k, k, n, stream=s, check=False)  # noqa: E731
    with torch.cuda.stream(s):
        res["mx_warm_up"] = mcall()
    s.synchronize()
    g_mx, res["mx_capture"] = capture(mcall, s)
    big = 8192
    bA = torch.zeros((big, big), dtype=torch.uint8, device="cuda")
    bS = torch.full((big, big // 32), 127, dtype=torch.uint8, device="cuda")
    bC = torch.empty((big, big), dtype=torch.bfloat16, device="cuda")
    res["big_mx"] = G.gemm_mxfp8(bA, bS, bA.clone(), bS.clone(), bC, big, big, big, big, big, big, check=False)
    torch.cuda.synchronize()
    a_c2, sfa2, b_c2, sfb2 = synth.mxfp8_operands(m, n, k, workload=413)
    dA.copy_(torch.from_numpy(a_c2))
    dB.copy_(torch.from_numpy(b_c2))
    dsa.copy_(torch.from_numpy(sfa2))
    dsb.copy_(torch.from_numpy(sfb2))
    g_mx.replay()
    torch.cuda.synchronize()
    c_ref, s_abs = oracle.gemm_mxfp8_f64(a_c2, sfa2, b_c2, sfb2, with_abs=True)
    got = Cm.cpu().float().numpy().astype(np.float64)
    res["mx_replay_max_excess"] = float(np.max(np.abs(got - c_ref) - (1e-3 * s_abs + 1e-6 + 2.0 ** -8 * np.abs(c_ref))))
    res["status"] = G.gemm_check_device_status(check=False)
    return res


if __name__ == "__main__":
    torch.cuda.set_device(0)
    case = sys.argv[1]
    print(json.dumps({"refuse_then_replay": refuse_then_replay,
                      "growth_after_capture": growth_after_capture}[case]()))
