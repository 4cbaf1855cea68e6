"""gemm_bf16_allgather: a row slab of C = A.B written by one kernel into
several copies of C (on a GPU node: this GPU's C and the other GPUs' mapped
C buffers).  On the one GPU here the destinations are separate local
buffers, which exercises the same kernel path: every destination must hold
the slab, bit-exact on integer inputs, and nothing outside the slab's rows
and columns may be touched."""
import numpy as np
import pytest
import torch

import oracle
from dense_gemm_engineering_bf16_b200 import gemm as G
from dense_gemm_engineering_bf16_b200 import synth

from gpu_helpers import SENTINEL_BF16, SENTINEL_F32, assert_close, assert_exact, to_device_bf16

pytestmark = pytest.mark.gpu


def _dest(M_total, ldc, c_type):
    if c_type == G.OUT_F32:
        host = np.full(M_total * ldc, SENTINEL_F32, dtype=np.uint32).view(np.int32)
    else:
        host = np.full(M_total * ldc, SENTINEL_BF16, dtype=np.uint16).view(np.int16)
    return torch.from_numpy(host).cuda()


def _read(t, M_total, ldc, c_type):
    if c_type == G.OUT_F32:
        bits = t.cpu().numpy().view(np.uint32).reshape(M_total, ldc)
        return bits, bits.view(np.float32).astype(np.float64), SENTINEL_F32
    bits = t.cpu().numpy().view(np.uint16).reshape(M_total, ldc)
    return bits, oracle.decode_bf16(bits), SENTINEL_BF16


@pytest.mark.parametrize("c_type", [G.OUT_F32, G.OUT_BF16])
@pytest.mark.parametrize("n_dst", [1, 3, 8])
@pytest.mark.parametrize("dist", ["ints", "normal"])
def test_slab_reaches_every_copy_of_c(c_type, n_dst, dist):
    M_total, row0, M, N, K = 1500, 384, 700, 900, 520
    ldc = N + (-N % 8) + 8                 # 16-byte rows for fp32 and bf16, with spare columns
    a_bits, b_bits = synth.bf16_operands(M, N, K, dist, workload=140, lda=K + 8, ldb=K + 8)
    A, B = to_device_bf16(a_bits), to_device_bf16(b_bits)
    dst = [_dest(M_total, ldc, c_type) for _ in range(n_dst)]
    G.gemm_bf16_allgather(A, B, dst, M, N, K, K + 8, K + 8, ldc, row0, c_type)
    G.gemm_check_device_status()
    c_ref, s_abs = oracle.gemm_bf16_f64(a_bits, b_bits, K=K, with_abs=True)
    for d, t in enumerate(dst):
        bits, vals, sentinel = _read(t, M_total, ldc, c_type)
        got = vals[row0:row0 + M, :N]
        if dist == "ints":
            assert_exact(got, c_ref, c_type, f"copy {d}")
        else:
            assert_close(got, c_ref, s_abs, c_type, f"copy {d}")
        outside = np.ones((M_total, ldc), bool)
        outside[row0:row0 + M, :N] = False
        assert np.all(bits[outside] == sentinel), f"copy {d}: write outside the slab"


def test_k_zero_writes_zeros_to_every_copy():
    M_total, row0, M, N = 600, 256, 200, 136
    dst = [_dest(M_total, N, G.OUT_F32) for _ in range(2)]
    A = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    G.gemm_bf16_allgather(A, A, dst, M, N, 0, 8, 8, N, row0, G.OUT_F32)
    G.gemm_check_device_status()
    for t in dst:
        bits, vals, sentinel = _read(t, M_total, N, G.OUT_F32)
        assert np.all(vals[row0:row0 + M] == 0)
        assert np.all(bits[:row0] == sentinel) and np.all(bits[row0 + M:] == sentinel)


def test_matches_gemm_bf16_on_the_slab():
    """The same slab through gemm_bf16 (into a slab-sized C) and through the
    all-gather entry point: identical bits (same kernel family and order)."""
    M, N, K = 1024, 2048, 1024
    a_bits, b_bits = synth.bf16_operands(M, N, K, "normal", workload=141)
    A, B = to_device_bf16(a_bits), to_device_bf16(b_bits)
    ref = torch.empty((M, N), dtype=torch.float32, device="cuda")
    G.gemm_force_config("2cta_256x256_clc")
    try:
        G.gemm_bf16(A, B, ref, M, N, K, K, K, N)
    finally:
        G.gemm_force_config("auto")
    dst = [torch.empty((4 * M, N), dtype=torch.float32, device="cuda") for _ in range(2)]
    G.gemm_bf16_allgather(A, B, dst, M, N, K, K, K, N, 2 * M)
    G.gemm_check_device_status()
    for t in dst:
        assert torch.equal(t[2 * M:3 * M], ref)


def test_argument_checks():
    A = torch.empty((64, 64), dtype=torch.bfloat16, device="cuda")
    C = torch.empty((256, 64), dtype=torch.float32, device="cuda")
    ptr = C.data_ptr()
    bad = {
        "no destination": [],
        "nine destinations": [ptr] * 9,
        "overlapping slabs": [ptr, ptr],
        "misaligned": [ptr + 4],
    }
    want = {"no destination": 1, "nine destinations": 1, "overlapping slabs": 3, "misaligned": 2}
    for name, dsts in bad.items():
        st = G.gemm_bf16_allgather(A, A, dsts, 64, 64, 64, 64, 64, 64, 0, check=False)
        assert st == want[name], (name, st)
    assert G.gemm_bf16_allgather(A, A, [ptr], 64, 64, 64, 64, 64, 64, -1, check=False) == 1
