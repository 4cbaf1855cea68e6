"""GPU parity of gemm_mxfp8 (E4M3 operands, one E8M0 scale per 32 K
elements, bf16 output) against the oracle, through the C ABI.

Bit-exact where every partial sum is exactly representable in fp32
(integer-valued elements, scales within a few binades); otherwise
|C - C_ref| <= 1e-3 sum|a b| + 1e-6 + 2^-8 |C_ref| (bf16 output).
The 8192^3 workload (scale exponents uniform in [-4, 4]) is checked on
sampled elements and, for every element, through row and column sums.
"""
import numpy as np
import pytest

import oracle
from dense_gemm_engineering_bf16_b200 import gemm as G
from dense_gemm_engineering_bf16_b200 import synth

from gpu_helpers import assert_close, assert_exact, run_mxfp8, sample_indices

pytestmark = pytest.mark.gpu
BF16 = G.OUT_BF16
MX_CFGS = ["mxfp8_1cta_128x256", "mxfp8_2cta_256x256"]


def _int_operands(M, N, K, seed, exp_lo=0, exp_hi=0):
    a = synth.to_e4m3_codes(synth.small_ints(seed, (M, K)))
    b = synth.to_e4m3_codes(synth.small_ints(seed + 1, (N, K)))
    sfa = (127 + synth.small_ints(seed + 2, (M, K // 32), exp_lo, exp_hi)).astype(np.uint8)
    sfb = (127 + synth.small_ints(seed + 3, (N, K // 32), exp_lo, exp_hi)).astype(np.uint8)
    return a, sfa, b, sfb


def _check(a, sfa, b, sfb, M, N, K, exact=False, ldc=None, cfg="auto"):
    C = run_mxfp8(a, sfa, b, sfb, M, N, K, ldc=ldc, config=cfg)
    got, guard_ok = C.download()
    assert guard_ok, "write outside C's M x N window"
    c_ref, s_abs = oracle.gemm_mxfp8_f64(a, sfa, b, sfb, K=K, with_abs=True)
    if exact:
        assert_exact(got, c_ref, BF16, f"mxfp8 {M}x{N}x{K}")
    else:
        assert_close(got, c_ref, s_abs, BF16, f"mxfp8 {M}x{N}x{K}")


@pytest.mark.parametrize("cfg", MX_CFGS)
def test_single_tile_unit_scales_bit_exact(cfg):
    _check(*_int_operands(128, 256, 128, seed=1), 128, 256, 128, exact=True, cfg=cfg)


@pytest.mark.parametrize("cfg", MX_CFGS)
def test_scaled_integers_bit_exact(cfg):
    # exponents in [-1, 1]: every partial sum is a multiple of 2^-2 below 2^22
    M, N, K = 256, 512, 1024
    _check(*_int_operands(M, N, K, seed=5, exp_lo=-1, exp_hi=1), M, N, K, exact=True, cfg=cfg)


@pytest.mark.parametrize("cfg", MX_CFGS)
def test_random_values_and_scales_multi_tile(cfg):
    M, N, K = 640, 768, 1024
    a, sfa, b, sfb = synth.mxfp8_operands(M, N, K, workload=40)
    _check(a, sfa, b, sfb, M, N, K, cfg=cfg)


@pytest.mark.parametrize("cfg", MX_CFGS)
@pytest.mark.parametrize("shape", [(1, 8, 32), (3, 5, 32), (127, 129, 96), (200, 300, 160),
                                   (129, 257, 64), (300, 40, 544), (1, 1000, 256), (257, 513, 4000)],
                         ids=lambda s: "x".join(map(str, s)))
def test_ragged_tails(shape, cfg):
    M, N, K = shape
    K = K // 32 * 32
    a, sfa, b, sfb = synth.mxfp8_operands(M, N, K, workload=41 + M)
    _check(a, sfa, b, sfb, M, N, K, cfg=cfg)


def test_strided_operands():
    M, N, K = 150, 260, 192
    a, sfa, b, sfb = synth.mxfp8_operands(M, N, K, workload=45)
    a_pad = np.full((M, 224), 0x7F, np.uint8)     # padding bytes are E4M3 NaN
    a_pad[:, :K] = a
    b_pad = np.full((N, 208), 0x7F, np.uint8)
    b_pad[:, :K] = b
    C = run_mxfp8(a_pad, sfa, b_pad, sfb, M, N, K, ldc=272)
    got, guard_ok = C.download()
    assert guard_ok
    c_ref, s_abs = oracle.gemm_mxfp8_f64(a, sfa, b, sfb, with_abs=True)
    assert_close(got, c_ref, s_abs, BF16, "strided")


def test_k_zero_writes_zeros():
    a = np.zeros((40, 16), np.uint8)
    b = np.zeros((50, 16), np.uint8)
    s = np.zeros((1, 1), np.uint8)
    C = run_mxfp8(a, s, b, s, 40, 50, 0)
    got, guard_ok = C.download()
    assert guard_ok and np.all(got == 0)


@pytest.mark.parametrize("cfg", MX_CFGS)
def test_nan_scale_poisons_its_block_only(cfg):
    M, N, K = 130, 140, 128
    a, sfa, b, sfb = synth.mxfp8_operands(M, N, K, workload=46)
    sfa[7, 2] = 0xFF
    C = run_mxfp8(a, sfa, b, sfb, M, N, K, config=cfg)
    got, _ = C.download()
    c_ref, s_abs = oracle.gemm_mxfp8_f64(a, sfa, b, sfb, with_abs=True)
    assert np.isnan(got[7]).all() and not np.isnan(np.delete(got, 7, axis=0)).any()
    assert_close(got, c_ref, s_abs, BF16, "nan scale")


def test_rejects_k_not_multiple_of_32():
    assert G.lib.gemm_mxfp8(0x7F0000000000, 0x7F0000100000, 0x7F0000200000, 0x7F0000300000,
                            0x7F0000400000, 64, 64, 48, 48, 48, 64, 0) == 1


@pytest.mark.parametrize("cfg", ["auto", "mxfp8_1cta_128x256"])
def test_mxfp8_8192_cube(cfg):
    """8192^3 block-scaled: E4M3 U[-1,1], scale exponents U{-4..4}, bf16 out
    (auto = the CTA-pair kernel the benchmark times)."""
    M = N = K = 8192
    a, sfa, b, sfb = synth.mxfp8_operands(M, N, K, workload=8)
    C = run_mxfp8(a, sfa, b, sfb, M, N, K, config=cfg)
    got, guard_ok = C.download()
    assert guard_ok and np.isfinite(got).all()
    rows = sample_indices(M, 128, 40, seed=81)
    cols = sample_indices(N, 256, 40, seed=82)
    c_ref, s_abs = oracle.gemm_mxfp8_f64(a, sfa, b, sfb, rows=rows, cols=cols, with_abs=True)
    assert_close(got[np.ix_(rows, cols)], c_ref, s_abs, BF16, "mxfp8 8192 sampled")
    a64 = oracle.decode_mx_operand(a, sfa, K)
    b64 = oracle.decode_mx_operand(b, sfb, K)
    r, r_mag, cl, cl_mag = oracle.gemm_line_sums_f64(a64, b64)
    half_ulp = (2.0 ** -8) * np.abs(got)
    assert np.all(np.abs(got.sum(axis=1) - r) <= 1e-3 * r_mag + 1e-6 * N + half_ulp.sum(axis=1))
    assert np.all(np.abs(got.sum(axis=0) - cl) <= 1e-3 * cl_mag + 1e-6 * M + half_ulp.sum(axis=0))


def test_unaligned_scale_pointers_take_the_byte_path():
    """Scales may sit at any address: at K = 1024 (scale rows of 32 bytes) an
    offset of one byte forces the repack's byte-load path."""
    import torch
    M, N, K = 200, 300, 1024
    a, sfa, b, sfb = synth.mxfp8_operands(M, N, K, workload=47)

    def dev_off(x):
        buf = torch.zeros(x.size + 16, dtype=torch.uint8, device="cuda")
        buf[1:1 + x.size] = torch.from_numpy(np.ascontiguousarray(x).reshape(-1)).cuda()
        return buf, buf.data_ptr() + 1

    A = torch.from_numpy(a).cuda()
    B = torch.from_numpy(b).cuda()
    SA, pa = dev_off(sfa)
    SB, pb = dev_off(sfb)
    ldc = 312                                  # 624-byte rows: a multiple of 16
    C = torch.zeros((M, ldc), dtype=torch.bfloat16, device="cuda")
    G.gemm_mxfp8(A, pa, B, pb, C, M, N, K, K, K, ldc)
    G.gemm_check_device_status()
    got = oracle.decode_bf16(C.cpu().view(torch.int16).numpy().view(np.uint16))[:, :N]
    c_ref, s_abs = oracle.gemm_mxfp8_f64(a, sfa, b, sfb, with_abs=True)
    assert_close(got, c_ref, s_abs, BF16, "unaligned scales")
