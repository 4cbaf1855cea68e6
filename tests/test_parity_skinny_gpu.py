"""GPU parity of the skinny path (M <= 256, chosen by shape for M <= 32): A and B swapped so 128 rows of B
fill the MMA, stream-K over every SM, split tiles finished by the last
contributor in contributor order.  Compared with the oracle element by
element; integer inputs bit-exact."""
import numpy as np
import pytest

import oracle
from dense_gemm_engineering_bf16_b200 import gemm as G
from dense_gemm_engineering_bf16_b200 import synth

from gpu_helpers import assert_close, assert_exact, run_gemm

pytestmark = pytest.mark.gpu
F32, BF16 = G.OUT_F32, G.OUT_BF16


def _check(M, N, K, dist, workload, c_type=F32, lda=None, config="skinny", repeats=1):
    a_bits, b_bits = synth.bf16_operands(M, N, K, dist, workload=workload, lda=lda, ldb=lda)
    C = run_gemm(a_bits, b_bits, M, N, K, c_type=c_type, config=config, repeats=repeats)
    got, guard_ok = C.download()
    assert guard_ok, "write outside C's M x N window"
    c_ref, s_abs = oracle.gemm_bf16_f64(a_bits, b_bits, K=K, with_abs=True)
    if dist == "ints":
        assert_exact(got, c_ref, c_type, f"skinny {M}x{N}x{K}")
    else:
        assert_close(got, c_ref, s_abs, c_type, f"skinny {M}x{N}x{K}")
    return C


def test_auto_selects_skinny_for_small_m():
    assert G.gemm_select_config(16, 8192, 8192) == G.CONFIGS["skinny"]
    assert G.gemm_select_config(32, 2048, 8192) == G.CONFIGS["skinny"]
    assert G.gemm_select_config(32, 4096, 4096) == G.CONFIGS["skinny"]
    # past 32 rows the split-K tile kernel wins
    assert G.gemm_select_config(64, 8192, 8192) == G.CONFIGS["1cta_128x128_splitk"]


@pytest.mark.parametrize("c_type", [F32, BF16])
def test_single_tile_integers_bit_exact(c_type):
    _check(128, 128, 128, "ints", workload=101, c_type=c_type)


@pytest.mark.parametrize("shape", [(1, 1, 1), (1, 8, 8), (16, 128, 64), (17, 129, 63), (64, 300, 1000),
                                   (65, 257, 200), (128, 640, 520), (129, 255, 65), (200, 1000, 4000),
                                   (256, 384, 2048)], ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("c_type", [F32, BF16])
def test_tails_and_mpad_buckets(shape, c_type):
    M, N, K = shape
    _check(M, N, K, "normal", workload=110 + M, c_type=c_type, lda=K + (-K % 8))


@pytest.mark.parametrize("shape", [(16, 4096, 8192), (48, 2048, 4096), (100, 1280, 3000), (250, 512, 16384)],
                         ids=lambda s: "x".join(map(str, s)))
def test_stream_k_split_tiles_integers_bit_exact(shape):
    """Shapes whose tiles are split across 2-4 CTAs; integer inputs make any
    lost, doubled or misplaced partial visible bit for bit."""
    M, N, K = shape
    _check(M, N, K, "ints", workload=130 + M)


def test_skinny_16_8192_8192_auto():
    _check(16, 8192, 8192, "normal", workload=6, config="auto")


def test_deterministic_and_reusable_workspace():
    a_bits, b_bits = synth.bf16_operands(40, 3000, 5000, "normal", workload=140)
    first = run_gemm(a_bits, b_bits, 40, 3000, 5000, config="skinny").bits()
    # a different, larger problem in between grows and reuses the workspace
    _check(200, 4096, 4096, "ints", workload=141)
    again = run_gemm(a_bits, b_bits, 40, 3000, 5000, config="skinny", repeats=3).bits()
    assert np.array_equal(first, again)


def test_forcing_skinny_above_256_rows_is_rejected():
    a_bits, b_bits = synth.bf16_operands(300, 64, 64, "uniform", workload=142)
    with pytest.raises(G.GemmError):
        run_gemm(a_bits, b_bits, 300, 64, 64, config="skinny")


# ---- the cluster-split form (M <= 64 with enough 128-row tiles of B to keep
# most SMs streaming): K split over 2 or 4 CTAs per tile, partials summed in
# member order through distributed shared memory

CLUSTER_SHAPES = [(16, 4096, 1024), (40, 8192, 512), (1, 3100, 2048), (64, 6400, 768)]


@pytest.mark.parametrize("shape", CLUSTER_SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("c_type", [F32, BF16])
def test_cluster_split_integers_bit_exact(shape, c_type):
    M, N, K = shape
    _check(M, N, K, "ints", workload=600 + M, c_type=c_type)


@pytest.mark.parametrize("shape", CLUSTER_SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("c_type", [F32, BF16])
def test_cluster_split_normal(shape, c_type):
    M, N, K = shape
    _check(M, N, K, "normal", workload=620 + M, c_type=c_type)


def test_cluster_split_deterministic():
    """Member order, not arrival order, fixes the sum: repeated calls give
    the same bits."""
    M, N, K = 24, 4096, 2048
    a_bits, b_bits = synth.bf16_operands(M, N, K, "normal", workload=640)
    first = run_gemm(a_bits, b_bits, M, N, K, config="skinny").bits()
    for _ in range(3):
        assert (run_gemm(a_bits, b_bits, M, N, K, config="skinny").bits() == first).all()


def test_cluster_split_fused_epilogue_and_transposed_b():
    """alpha, beta, bias and ReLU in the owner's write-back; B stored K x N."""
    import torch

    from gpu_helpers import to_device_bf16
    M, N, K = 33, 4096, 1024
    a, b = synth.bf16_operands(M, N, K, "ints", workload=641)
    bT = np.ascontiguousarray(b.T)
    c_old = synth.small_ints(642, (M, N), -8, 8)
    bias = synth.small_ints(643, (N,), -20, 20).astype(np.float32)
    C = torch.from_numpy(c_old.astype(np.float32)).cuda()
    G.gemm_force_config("skinny")
    try:
        G.gemm_bf16_fused(to_device_bf16(a), to_device_bf16(bT), C, M, N, K, K, N, N, F32, G.KMAJOR, G.MNMAJOR,
                          1.0, -1.0, torch.from_numpy(bias).cuda(), G.ACT_RELU)
    finally:
        G.gemm_force_config("auto")
    G.gemm_check_device_status()
    ab = oracle.gemm_bf16_f64(a, b)
    want = oracle.epilogue(ab, c_old.astype(np.float64), 1.0, -1.0, bias.astype(np.float64), G.ACT_RELU)
    assert_exact(C.cpu().numpy().astype(np.float64), want, F32, "cluster skinny fused")
