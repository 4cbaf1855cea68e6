"""gemm_bf16_noalloc, the entry point for callers that cannot allocate device
memory (a framework's caching allocator owns the device, allocator callbacks
must not re-enter it, or cudaMalloc's implicit synchronisation is not
allowed).  Its kernels keep their scratch in a static array inside the
library instead of cudaMalloc'd memory.

This file is collected last on purpose: it must pass both alone in a fresh
process and after every other test.
"""
import numpy as np
import pytest
import torch

import oracle
from dense_gemm_engineering_bf16_b200 import gemm as G
from dense_gemm_engineering_bf16_b200 import synth

from gpu_helpers import tolerance, to_device_bf16

pytestmark = pytest.mark.gpu

# two calls in a row: different shapes through the same kernel instantiation
# (one-CTA 128 x 128 tiles; both products are past the latency path's bound),
# so the second call cannot trigger a first-use kernel load
CASES = [(600, 400, 1000, G.OUT_F32), (777, 1030, 1000, G.OUT_F32)]


def _decode(c, c_type):
    if c_type == G.OUT_F32:
        return c.cpu().numpy().astype(np.float64)
    return oracle.decode_bf16(c.cpu().view(torch.int16).numpy().view(np.uint16))


def test_noalloc_matches_gemm_bf16_on_two_calls_in_a_row():
    G.gemm_force_config("auto")
    prepared = []
    for i, (M, N, K, c_type) in enumerate(CASES):
        lda = K + (-K % 8)
        a_bits, b_bits = synth.bf16_operands(M, N, K, "normal", workload=70 + i, lda=lda, ldb=lda)
        dt = torch.float32 if c_type == G.OUT_F32 else torch.bfloat16
        ldc = N + (-N % 8)
        prepared.append(dict(M=M, N=N, K=K, c_type=c_type, lda=lda, ldc=ldc, a=a_bits, b=b_bits,
                             A=to_device_bf16(a_bits), B=to_device_bf16(b_bits),
                             C_na=torch.full((M, ldc), float("nan"), dtype=dt, device="cuda"),
                             C_ref=torch.full((M, ldc), float("nan"), dtype=dt, device="cuda")))
    torch.cuda.synchronize()

    # the allocation-free entry point, twice in a row; the second call must
    # not change the device's free memory (any cudaMalloc takes >= 2 MiB)
    free_before = None
    for i, p in enumerate(prepared):
        if i == 1:
            torch.cuda.synchronize()
            free_before = torch.cuda.mem_get_info()[0]
        G.gemm_bf16_noalloc(p["A"], p["B"], p["C_na"], p["M"], p["N"], p["K"], p["lda"], p["lda"],
                            p["ldc"], p["c_type"])
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before

    # the existing entry point on the same inputs
    for p in prepared:
        G.gemm_bf16(p["A"], p["B"], p["C_ref"], p["M"], p["N"], p["K"], p["lda"], p["lda"],
                    p["ldc"], p["c_type"])
    G.gemm_check_device_status()

    for p in prepared:
        M, N, K = p["M"], p["N"], p["K"]
        got = _decode(p["C_na"], p["c_type"])
        ref = _decode(p["C_ref"], p["c_type"])
        assert np.isnan(got[:, N:]).all(), "wrote past column N"
        got, ref = got[:, :N], ref[:, :N]
        c64, s_abs = oracle.gemm_bf16_f64(p["a"], p["b"], K=K, with_abs=True)
        tol = tolerance(c64, s_abs, p["c_type"])
        assert np.all(np.abs(got - ref) <= tol), f"{M}x{N}x{K}: differs from gemm_bf16"
        assert np.all(np.abs(got - c64) <= tol), f"{M}x{N}x{K}: outside the oracle tolerance"


def test_noalloc_runs_the_cluster_launch_control_kernel():
    """A shape of >= 148 pair tiles, where the shape choice is the CLC kernel:
    bit-identical to gemm_bf16 (same kernel, same order)."""
    M, N, K = 4096, 4608, 2304             # 288 pair tiles, K past the static schedule's range
    assert G.gemm_select_config(M, N, K) == G.CONFIGS["2cta_256x256_clc"]
    a_bits, b_bits = synth.bf16_operands(M, N, K, "normal", workload=73)
    A, B = to_device_bf16(a_bits), to_device_bf16(b_bits)
    C_ref = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    C_na = torch.empty_like(C_ref)
    G.gemm_bf16(A, B, C_ref, M, N, K, K, K, N, G.OUT_BF16)
    G.gemm_bf16_noalloc(A, B, C_na, M, N, K, K, K, N, G.OUT_BF16)
    G.gemm_check_device_status()
    assert torch.equal(C_ref, C_na)
    rows = np.arange(0, M, 61)
    c64, s_abs = oracle.gemm_bf16_f64(a_bits, b_bits, rows=rows, with_abs=True)
    got = _decode(C_na, G.OUT_BF16)[rows]
    assert np.all(np.abs(got - c64) <= tolerance(c64, s_abs, G.OUT_BF16))


@pytest.mark.parametrize("shape", [(16, 1024, 8192), (16, 8192, 4096)], ids=["split_k_tiles", "skinny_cluster"])
def test_noalloc_small_m_needs_no_workspace(shape):
    """Where gemm_bf16 takes the skinny kernel, the allocation-free entry
    point runs its cluster split (8192 columns: 64 tiles of B) or, where
    that does not apply (1024 columns), the split-K tile kernel: both sum
    their partials in shared memory.  Same result within the tolerance, no
    device memory taken."""
    M, N, K = shape
    assert G.gemm_select_config(M, N, K) == G.CONFIGS["skinny"]
    a_bits, b_bits = synth.bf16_operands(M, N, K, "normal", workload=74)
    A, B = to_device_bf16(a_bits), to_device_bf16(b_bits)
    C = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    G.gemm_bf16_noalloc(A, B, C, M, N, K, K, K, N, G.OUT_F32)     # first use of this kernel: loads it
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    C.fill_(float("nan"))
    G.gemm_bf16_noalloc(A, B, C, M, N, K, K, K, N, G.OUT_F32)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before
    G.gemm_check_device_status()
    c64, s_abs = oracle.gemm_bf16_f64(a_bits, b_bits, with_abs=True)
    got = C.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - c64) <= tolerance(c64, s_abs, G.OUT_F32))


def test_noalloc_argument_checks_match():
    ptr = 0x7F0000000000
    for args in [(-1, 8, 8, 8, 8, 8, 0), (8, 8, 8, 4, 8, 8, 0), (8, 8, 8, 8, 8, 8, 9)]:
        M, N, K, lda, ldb, ldc, ct = args
        assert G.lib.gemm_bf16_noalloc(ptr, ptr + 4096, ptr + 8192, M, N, K, lda, ldb, ldc, ct, 0) == \
            G.lib.gemm_bf16(ptr, ptr + 4096, ptr + 8192, M, N, K, lda, ldb, ldc, ct, 0)
