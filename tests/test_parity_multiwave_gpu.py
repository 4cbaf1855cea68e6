"""Element-by-element parity of the schedules that only run when tiles
outnumber the co-resident clusters, against the oracle, through the C ABI.

A persistent kernel's first wave and its later tiles take different code
paths: a static schedule strides (tile, tile + clusters, ...), and a Cluster
Launch Control (CLC) schedule cancels pending clusters and hands their tiles
to running ones.  With at most ~74 CTA pairs (or ~148 CTAs) resident, those
paths need more tiles than that, so every shape here has several waves of
tiles for every configuration, while K stays short enough for the oracle to
check every element in seconds.  This is the validation procedure of "GPU
执行模型", section "验证流程": a small-shape reference first, then the
maximum shapes (the full 8192^3 comparison closes this file).

Tile counts at 4096 x 4864:
  512 x 256 (two-consumer pair)  8 x 19 =  152 tiles
  256 x 256 (pair)              16 x 19 =  304
  128 x 256 (one CTA)           32 x 19 =  608
  128 x 128 (one CTA)           32 x 38 = 1216
"""
import functools

import numpy as np
import pytest

import oracle
from dense_gemm_engineering_bf16_b200 import gemm as G
from dense_gemm_engineering_bf16_b200 import synth

from gpu_helpers import assert_close, assert_exact, run_gemm, run_mxfp8

pytestmark = pytest.mark.gpu

CFGS = ["1cta_128x128", "1cta_128x256", "2cta_256x256", "1cta_128x256_clc", "2cta_256x256_clc", "2cta_512x256_clc",
        "2cta_256x256_sk", "2cta_256x224"]
F32, BF16 = G.OUT_F32, G.OUT_BF16
WAVES = (4096, 4864, 256)


@functools.lru_cache(maxsize=4)
def _case(M, N, K, dist, workload, with_abs):
    """Seeded operands and the oracle's result, shared by the configurations."""
    a_bits, b_bits = synth.bf16_operands(M, N, K, dist, workload=workload)
    ref = oracle.gemm_bf16_f64(a_bits, b_bits, K=K, with_abs=with_abs)
    return a_bits, b_bits, ref


def _tiles(cfg, M, N):
    bm, bn = {"1cta_128x128": (128, 128), "1cta_128x256": (128, 256), "2cta_256x256": (256, 256),
              "1cta_128x256_clc": (128, 256), "2cta_256x256_clc": (256, 256), "2cta_512x256_clc": (512, 256),
              "2cta_256x256_sk": (256, 256), "2cta_256x224": (256, 224)}[cfg]
    pair = cfg.startswith("2cta")
    return -(-M // bm) * -(-N // bn), (74 if pair else 148)


@pytest.mark.parametrize("c_type", [F32, BF16])
@pytest.mark.parametrize("cfg", CFGS)
def test_several_waves_integers_bit_exact(cfg, c_type):
    """Small integers: every partial sum is an exact fp32 integer, so every
    element must equal the oracle's single rounding, in every wave."""
    M, N, K = WAVES
    tiles, resident = _tiles(cfg, M, N)
    assert tiles > resident, "the shape must need more than one wave"
    a_bits, b_bits, c_ref = _case(M, N, K, "ints", 110, False)
    C = run_gemm(a_bits, b_bits, M, N, K, c_type=c_type, config=cfg)
    got, guard_ok = C.download()
    assert guard_ok, "write outside C's M x N window"
    assert_exact(got, c_ref, c_type, f"{cfg} {M}x{N}x{K}")


@pytest.mark.parametrize("cfg", CFGS)
def test_several_waves_ragged_normal(cfg):
    """4000 x 3000 x 2000 (the ragged workload's shape and K tail) forced onto
    every configuration: 96 two-consumer tiles, 192 pair tiles, 384 / 768
    one-CTA tiles, each more than one wave; N(0,1) inputs, every element."""
    M, N, K = 4000, 3000, 2000
    tiles, resident = _tiles(cfg, M, N)
    assert tiles > resident
    a_bits, b_bits, (c_ref, s_abs) = _case(M, N, K, "normal", 4, True)
    C = run_gemm(a_bits, b_bits, M, N, K, config=cfg)
    got, guard_ok = C.download()
    assert guard_ok
    assert_close(got, c_ref, s_abs, F32, f"{cfg} {M}x{N}x{K}")


@pytest.mark.parametrize("cfg", ["2cta_512x256_clc", "2cta_256x256_clc", "2cta_256x256_sk"])
def test_several_waves_repeat_identical(cfg):
    """A CLC schedule assigns tiles to pairs by timing, differently on every
    run; the per-element order is fixed by the tile, so results must not
    change from run to run."""
    M, N, K = WAVES
    a_bits, b_bits = synth.bf16_operands(M, N, K, "normal", workload=111)
    first = run_gemm(a_bits, b_bits, M, N, K, config=cfg).bits()
    again = run_gemm(a_bits, b_bits, M, N, K, config=cfg, repeats=3).bits()
    assert np.array_equal(first, again)


# --------------------------------------------------------------- MXFP8 --

def _mx_int_operands(M, N, K, seed):
    a = synth.to_e4m3_codes(synth.small_ints(seed, (M, K)))
    b = synth.to_e4m3_codes(synth.small_ints(seed + 1, (N, K)))
    sfa = np.full((M, K // 32), 127, np.uint8)
    sfb = np.full((N, K // 32), 127, np.uint8)
    return a, sfa, b, sfb


@pytest.mark.parametrize("cfg", ["mxfp8_1cta_128x256", "mxfp8_2cta_256x256"])
def test_mxfp8_several_waves_integers_bit_exact(cfg):
    """608 one-CTA tiles or 304 pair tiles, unit scales, integer elements."""
    M, N, K = WAVES
    a, sfa, b, sfb = _mx_int_operands(M, N, K, seed=120)
    C = run_mxfp8(a, sfa, b, sfb, M, N, K, config=cfg)
    got, guard_ok = C.download()
    assert guard_ok
    c_ref = oracle.gemm_mxfp8_f64(a, sfa, b, sfb, K=K)
    assert_exact(got, c_ref, BF16, f"{cfg} {M}x{N}x{K}")


@pytest.mark.parametrize("cfg", ["mxfp8_1cta_128x256", "mxfp8_2cta_256x256"])
def test_mxfp8_several_waves_scaled(cfg):
    """The workload's recipe (E4M3 U[-1,1], scale exponents U{-4..4}) at
    several waves and a K of four scale blocks per k-tile: every element."""
    M, N, K = 4000, 4864, 512
    a, sfa, b, sfb = synth.mxfp8_operands(M, N, K, workload=121)
    C = run_mxfp8(a, sfa, b, sfb, M, N, K, config=cfg)
    got, guard_ok = C.download()
    assert guard_ok
    c_ref, s_abs = oracle.gemm_mxfp8_f64(a, sfa, b, sfb, K=K, with_abs=True)
    assert_close(got, c_ref, s_abs, BF16, f"{cfg} {M}x{N}x{K}")


# ------------------------------------------------------- maximum shape --

def test_square_8192_every_element():
    """The headline problem (8192^3, U[-1,1], fp32 out) in the configuration
    the benchmark times, compared with the oracle on all 67M elements.  The
    tolerance scale sum_k |a_ik b_kj| is |A| |B| (an fp64 library product;
    it only sizes the tolerance)."""
    M = N = K = 8192
    assert G.gemm_select_config(M, N, K) == G.CONFIGS["2cta_512x256_clc"]
    a_bits, b_bits = synth.bf16_operands(M, N, K, "uniform", workload=3)
    C = run_gemm(a_bits, b_bits, M, N, K)
    got, guard_ok = C.download()
    del C
    assert guard_ok
    c_ref = oracle.gemm_bf16_f64(a_bits, b_bits, K=K)
    a_abs = np.abs(oracle.decode_bf16(a_bits))
    b_abs = np.abs(oracle.decode_bf16(b_bits))
    s_abs = a_abs @ b_abs.T
    del a_abs, b_abs
    assert_close(got, c_ref, s_abs, F32, "8192^3 every element")
