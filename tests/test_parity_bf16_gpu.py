"""GPU parity of gemm_bf16 against the oracle, through the C ABI.

Every config of the dense bf16 workload set is covered: the single 128^3 tile
(uniform and small-integer inputs), the 4096^3 square with fp32 and bf16
outputs, the 8192^3 headline square in the launch configuration the
benchmark times, and the ragged / skinny shapes.  Small shapes are compared
element by element; full-size shapes on sampled elements (every tile
boundary plus random ones) and, for every element at once, through the row-
and column-sum identity of the product.  Guard bands around C catch stray
writes.
"""
import numpy as np
import pytest
import torch

import oracle
from dense_gemm_engineering_bf16_b200 import gemm as G
from dense_gemm_engineering_bf16_b200 import synth

from gpu_helpers import (assert_close, assert_exact, run_gemm, sample_indices)

pytestmark = pytest.mark.gpu

CFGS = ["1cta_128x128", "1cta_128x256", "2cta_256x256", "1cta_128x256_clc", "2cta_256x256_clc", "2cta_512x256_clc",
        "2cta_256x256_sk", "2cta_256x224", "1cta_128x128_splitk", "1cta_128x256_splitk"]
F32, BF16 = G.OUT_F32, G.OUT_BF16


def _full_check(M, N, K, dist, workload, cfg="auto", c_type=F32, lda=None, ldb=None, ldc=None):
    a_bits, b_bits = synth.bf16_operands(M, N, K, dist, workload=workload, lda=lda, ldb=ldb)
    C = run_gemm(a_bits, b_bits, M, N, K, c_type=c_type, ldc=ldc, config=cfg)
    got, guard_ok = C.download()
    assert guard_ok, "write outside C's M x N window"
    c_ref, s_abs = oracle.gemm_bf16_f64(a_bits, b_bits, K=K, with_abs=True)
    if dist == "ints":
        assert_exact(got, c_ref, c_type, f"{cfg} {M}x{N}x{K}")
    else:
        assert_close(got, c_ref, s_abs, c_type, f"{cfg} {M}x{N}x{K}")
    return C


# ------------------------------------------------- single tile (128^3) --

@pytest.mark.parametrize("cfg", CFGS)
def test_single_tile_small_integers_bit_exact(cfg):
    _full_check(128, 128, 128, "ints", workload=1, cfg=cfg)


@pytest.mark.parametrize("cfg", CFGS)
def test_single_tile_uniform(cfg):
    _full_check(128, 128, 128, "uniform", workload=1, cfg=cfg)


# ------------------------------------------- several tiles, K loop, outs --

@pytest.mark.parametrize("cfg", CFGS)
@pytest.mark.parametrize("c_type", [F32, BF16])
def test_multi_tile_k_loop(cfg, c_type):
    _full_check(512, 768, 1024, "normal", workload=20, cfg=cfg, c_type=c_type)


@pytest.mark.parametrize("cfg", CFGS)
@pytest.mark.parametrize("c_type", [F32, BF16])
def test_integers_bit_exact_many_tiles(cfg, c_type):
    _full_check(640, 1024, 1536, "ints", workload=21, cfg=cfg, c_type=c_type)


# ------------------------------------------------------ tails and edges --

TAIL_SHAPES = [(1, 1, 1), (1, 8, 8), (127, 129, 63), (129, 255, 65), (257, 511, 200),
               (300, 40, 17), (33, 300, 1000), (255, 257, 64)]


@pytest.mark.parametrize("cfg", CFGS)
@pytest.mark.parametrize("shape", TAIL_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_ragged_tails(cfg, shape):
    M, N, K = shape
    lda = K + (-K % 8)               # 16-byte row pitch; the pad columns hold NaN patterns
    _full_check(M, N, K, "normal", workload=30 + M, cfg=cfg, lda=lda, ldb=lda)


@pytest.mark.parametrize("cfg", CFGS)
def test_strided_leading_dimensions(cfg):
    _full_check(300, 200, 136, "uniform", workload=40, cfg=cfg, lda=200, ldb=160, ldc=264)


def test_k_zero_writes_zeros():
    a = np.zeros((70, 8), np.uint16)
    b = np.zeros((90, 8), np.uint16)
    for c_type in (F32, BF16):
        C = run_gemm(a, b, 70, 90, 0, c_type=c_type)
        got, guard_ok = C.download()
        assert guard_ok and np.all(got == 0) and not np.signbit(got).any()


def test_empty_m_or_n_touches_nothing():
    a = np.zeros((4, 8), np.uint16)
    for M, N in ((0, 16), (16, 0)):
        C = run_gemm(a, a, M, N, 8)
        _, guard_ok = C.download()
        assert guard_ok


@pytest.mark.parametrize("cfg", ["auto", "1cta_128x128", "2cta_256x256", "2cta_256x256_clc", "2cta_512x256_clc",
                                 "1cta_128x128_splitk", "skinny"])
def test_nan_and_inf_propagate(cfg):
    """A NaN in A (row 17) and in B (column 250) makes that row and column of
    C NaN; an infinity in A (row 40) makes row 40 an infinity with the sign of
    the B element it meets, exactly as the oracle's IEEE arithmetic does.
    ("auto" takes the latency path at this size.)"""
    M, N, K = 200, 300, 256
    a_bits, b_bits = synth.bf16_operands(M, N, K, "uniform", workload=50)
    a_bits[17, 100] = 0x7FC0
    b_bits[250, 3] = 0x7FC0
    a_bits[40, 7] = 0x7F80
    C = run_gemm(a_bits, b_bits, M, N, K, config=cfg)
    got, guard_ok = C.download()
    assert guard_ok
    c_ref, s_abs = oracle.gemm_bf16_f64(a_bits, b_bits, with_abs=True)
    assert np.array_equal(np.isinf(got), np.isinf(c_ref)), f"{cfg}: infinity pattern differs"
    inf = np.isinf(c_ref)
    assert np.array_equal(np.sign(got[inf]), np.sign(c_ref[inf])), f"{cfg}: infinity signs differ"
    assert inf[40].sum() > 250, "the infinite row is row 40"
    fin = ~inf
    assert_close(np.where(fin, got, 0.0), np.where(fin, c_ref, 0.0), np.where(fin, s_abs, 0.0), F32,
                 f"{cfg}: nan")


@pytest.mark.parametrize("cfg", CFGS)
def test_deterministic(cfg):
    a_bits, b_bits = synth.bf16_operands(700, 600, 2000, "normal", workload=60)
    c1 = run_gemm(a_bits, b_bits, 700, 600, 2000, config=cfg).bits()
    c2 = run_gemm(a_bits, b_bits, 700, 600, 2000, config=cfg, repeats=3).bits()
    assert np.array_equal(c1, c2)


# ----------------------------------------------------- workload configs --

def _big_check(M, N, K, dist, workload, c_type=F32, cfg="auto", n_extra=40):
    """Full-size run: sampled elements vs the oracle one by one, and every
    element through the row / column sums of C."""
    a_bits, b_bits = synth.bf16_operands(M, N, K, dist, workload=workload)
    C = run_gemm(a_bits, b_bits, M, N, K, c_type=c_type, config=cfg)
    got, guard_ok = C.download()
    assert guard_ok
    assert np.isfinite(got).all()
    rows = sample_indices(M, 128, n_extra, seed=workload)
    cols = sample_indices(N, 128, n_extra, seed=workload + 7)
    c_ref, s_abs = oracle.gemm_bf16_f64(a_bits, b_bits, rows=rows, cols=cols, with_abs=True)
    assert_close(got[np.ix_(rows, cols)], c_ref, s_abs, c_type, f"{M}x{N}x{K} sampled")
    a64 = oracle.decode_bf16(a_bits)
    b64 = oracle.decode_bf16(b_bits)
    r, r_mag, cl, cl_mag = oracle.gemm_line_sums_f64(a64, b64)
    extra = (2.0 ** -8) * np.abs(got) if c_type == BF16 else 0.0
    row_tol = 1e-3 * r_mag + 1e-6 * N + (extra.sum(axis=1) if c_type == BF16 else 0.0)
    col_tol = 1e-3 * cl_mag + 1e-6 * M + (extra.sum(axis=0) if c_type == BF16 else 0.0)
    assert np.all(np.abs(got.sum(axis=1) - r) <= row_tol), "row sums"
    assert np.all(np.abs(got.sum(axis=0) - cl) <= col_tol), "column sums"


@pytest.mark.parametrize("c_type", [F32, BF16])
def test_square_4096(c_type):
    _big_check(4096, 4096, 4096, "normal_scaled", workload=2, c_type=c_type)


def test_square_8192_headline_launch():
    """8192^3, U[-1,1], fp32 out, the shape-selected (benchmark) configuration:
    512 x 256 pair tiles, two MMA consumers, Cluster Launch Control."""
    assert G.gemm_select_config(8192, 8192, 8192) == G.CONFIGS["2cta_512x256_clc"]
    _big_check(8192, 8192, 8192, "uniform", workload=3)


@pytest.mark.parametrize("cfg", ["2cta_256x256_clc", "1cta_128x256_clc", "2cta_512x256_clc"])
def test_square_8192_cluster_launch_control(cfg):
    """8192^3 with tiles handed out by Cluster Launch Control: 1024 (pair) or
    2048 (single) clusters launched, ~74 / 148 running at a time."""
    _big_check(8192, 8192, 8192, "uniform", workload=3, cfg=cfg)


def test_ragged_4000_3000_2000_full():
    _full_check(4000, 3000, 2000, "normal", workload=4)


def test_skinny_1000_8192_8192():
    _big_check(1000, 8192, 8192, "normal", workload=5)


def test_skinny_16_8192_8192_full():
    _full_check(16, 8192, 8192, "normal", workload=6)
