"""Pins for the oracle: each checks it against something other than itself --
a value the pages print, a closed form, an invariant, exact integer or
rational arithmetic, or an independent decoder.  CPU only.

A plausible mistake anywhere in the oracle (a dropped term, a wrong sign or
index, a transposed operand, a wrong scale block, double rounding) fails at
least one of these.
"""
import itertools
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from dense_gemm_engineering_bf16_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_kv(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split("=")
            out[k] = int(v)
    return out


# ---------------------------------------------------------------- ledger --

def test_tile_ledger_worked_example():
    """"GPU 执行模型", section "Tile 小账本": (64,64,32), 2 B, 2 stages, 48 KiB."""
    g = _read_kv("tile_ledger_worked_example.txt")
    led = oracle.gemm_tile_ledger(g["m_tile"], g["n_tile"], g["k_tile"],
                                  g["element_bytes"], g["stages"], g["smem_limit"])
    assert led.smem_bytes == g["smem_bytes"]
    assert led.flops == g["flops"]
    assert led.hbm_bytes == g["hbm_bytes"]
    assert led.arithmetic_intensity == g["arithmetic_intensity"]
    assert led.fits_smem == bool(g["fits_smem"])


def test_tile_ledger_matches_capacity_estimate_and_invariants():
    """The capacity estimate 2s(M_t K_t + K_t N_t) of section "Tile 的容量约束"
    equals the ledger's ring size for 2-byte elements; stages scale residency
    but not HBM bytes; one multiply-add is 2 FLOPs."""
    for m, n, k, s in [(64, 64, 32, 2), (128, 256, 64, 4), (256, 256, 64, 6), (16, 8, 8, 1)]:
        led = oracle.gemm_tile_ledger(m, n, k, 2, s, 227 << 10)
        assert led.smem_bytes == oracle.smem_estimate_double_buffer(m, n, k, s)
        led1 = oracle.gemm_tile_ledger(m, n, k, 2, 1, 227 << 10)
        assert led.hbm_bytes == led1.hbm_bytes
        assert led.smem_bytes == s * led1.smem_bytes
        assert led.flops == 2 * m * n * k
    # the 2-CTA pair stage of the big config: 256x256x64 bf16 -> AI 128
    assert oracle.gemm_tile_ledger(256, 256, 64, 2, 1, 1 << 30).arithmetic_intensity == 128
    assert not oracle.gemm_tile_ledger(64, 64, 32, 2, 4, 16383).fits_smem
    with pytest.raises(ValueError):
        oracle.gemm_tile_ledger(64, 0, 32, 2, 2, 1)


# ---------------------------------------------------------------- codecs --

def test_bf16_decode_all_codes_matches_torch():
    codes = np.arange(1 << 16, dtype=np.uint16)
    ours = oracle.decode_bf16(codes)
    ref = torch.from_numpy(codes.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))


def test_e4m3_decode_all_codes_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.decode_e4m3(codes)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert nan.sum() == 2 and np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9


def test_e8m0_decode_closed_form():
    assert oracle.decode_e8m0(127) == 1.0
    assert oracle.decode_e8m0(0) == 2.0 ** -127
    assert oracle.decode_e8m0(254) == 2.0 ** 127
    assert oracle.decode_e8m0(131) == 16.0 and oracle.decode_e8m0(123) == 1.0 / 16
    assert np.isnan(oracle.decode_e8m0(255))


def test_bf16_rounding_agrees_with_torch_on_binary32_values():
    """For values already representable in binary32 there is no double
    rounding, so torch's float -> bfloat16 (RNE) is an independent check."""
    rng = np.random.default_rng(7)
    x32 = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(5000) * 1e-39).astype(np.float32),   # bf16 subnormal range
        (rng.standard_normal(5000) * 1e-38).astype(np.float32),
        (rng.standard_normal(5000) * 1e-41).astype(np.float32),   # rounds to zero
        (rng.standard_normal(5000) * 1e37).clip(-3e38, 3e38).astype(np.float32),  # near overflow
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.4e38, np.inf, -np.inf], dtype=np.float32),
    ])
    ours = oracle.round_bf16(x32.astype(np.float64))
    ref = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_rounding_ties_and_no_double_rounding():
    one = 0x3F80
    # exact tie between 1 and 1+2^-7 -> even (1.0)
    assert oracle.f64_to_bf16_bits(1 + 2.0 ** -8) == one
    # tie between 1+2^-7 (odd) and 1+2^-6 (even) -> 1+2^-6
    assert oracle.f64_to_bf16_bits(1 + 3 * 2.0 ** -8) == one + 2
    # just above the tie: must round up.  Via binary32 the 2^-40 would be lost
    # and the tie would then round down -- the oracle rounds fp64 directly.
    assert oracle.f64_to_bf16_bits(1 + 2.0 ** -8 + 2.0 ** -40) == one + 1
    assert oracle.f64_to_bf16_bits(-(1 + 2.0 ** -8 + 2.0 ** -40)) == 0x8000 | (one + 1)
    # overflow and the largest finite value
    assert oracle.f64_to_bf16_bits(2.0 ** 128) == 0x7F80
    assert oracle.f64_to_bf16_bits((2 - 2.0 ** -7) * 2.0 ** 127) == 0x7F7F
    assert oracle.f64_to_bf16_bits(2.0 ** -133) == 0x0001        # smallest subnormal
    assert oracle.f64_to_bf16_bits(2.0 ** -134) == 0x0000        # tie to even (0)
    assert np.isnan(oracle.decode_bf16(np.array([oracle.f64_to_bf16_bits(float("nan"))], np.uint16))[0])


def test_f32_rounding_ties():
    r = oracle.round_f32(np.array([1 + 2.0 ** -24, 1 + 3 * 2.0 ** -24, 1 + 2.0 ** -24 + 2.0 ** -50,
                                   2.0 ** 128, -0.0]))
    assert r[0] == np.float32(1.0)
    assert r[1] == np.float32(1 + 2.0 ** -22)
    assert r[2] == np.float32(1 + 2.0 ** -23)
    assert np.isinf(r[3])
    assert np.signbit(r[4])


# ------------------------------------------------------------------ GEMM --

def _exact_gemm(a64, b64_nk):
    """Rational-arithmetic C = A.B with b(k,j) = B[j][k]: a second,
    independent formulation of the same definition."""
    M, K = a64.shape
    N = b64_nk.shape[0]
    fa = [[Fraction(float(v)) for v in row] for row in a64]
    fb = [[Fraction(float(v)) for v in row] for row in b64_nk]
    return [[sum((fa[i][k] * fb[j][k] for k in range(K)), Fraction(0)) for j in range(N)]
            for i in range(M)]


@pytest.mark.parametrize("dist", ["uniform", "ints", "normal"])
def test_brute_force_all_tiny_shapes(dist):
    """Every (M, N, K) in {1..5}^3 against exact rational arithmetic."""
    seed = 0
    for M, N, K in itertools.product(range(1, 6), repeat=3):
        seed += 1
        a_bits, b_bits = synth.bf16_operands(M, N, K, dist, workload=900 + seed)
        c, s = oracle.gemm_bf16_f64(a_bits, b_bits, with_abs=True)
        exact = _exact_gemm(oracle.decode_bf16(a_bits), oracle.decode_bf16(b_bits))
        for i in range(M):
            for j in range(N):
                # fp64 summation of <= 5 exact products: error below 2^-50 of sum|ab|
                assert abs(Fraction(c[i, j]) - exact[i][j]) <= Fraction(s[i, j]) * Fraction(1, 2 ** 50), \
                    (M, N, K, i, j)
                if dist != "normal":
                    assert Fraction(c[i, j]) == exact[i][j]


def test_small_integer_matrices_exact():
    """Integer inputs in [-4, 4]: the oracle is exact and equals integer arithmetic
    (pure Python ints, written out index by index)."""
    for (M, N, K) in [(7, 9, 13), (33, 17, 64), (128, 128, 128)]:
        a_bits, b_bits = synth.bf16_operands(M, N, K, "ints", workload=77)
        a = oracle.decode_bf16(a_bits).astype(np.int64)
        b = oracle.decode_bf16(b_bits).astype(np.int64)
        c = oracle.gemm_bf16_f64(a_bits, b_bits)
        for i in range(0, M, max(1, M // 9)):
            for j in range(0, N, max(1, N // 9)):
                want = 0
                for k in range(K):
                    want += int(a[i, k]) * int(b[j, k])
                assert c[i, j] == want
        assert np.array_equal(c, (a @ b.T).astype(np.float64))


def test_identity_and_permutations():
    M = K = 48
    N = 40
    a_bits, b_bits = synth.bf16_operands(M, N, K, "ints", workload=5)
    a = oracle.decode_bf16(a_bits)
    b = oracle.decode_bf16(b_bits)
    eye_bits = synth.to_bf16_bits(np.eye(K))
    # A = I  =>  C[i][j] = b(i, j) = B[j][i]
    c = oracle.gemm_bf16_f64(eye_bits, b_bits)
    assert np.array_equal(c, b.T)
    # B = I (stored N x K with N = K)  =>  C = A
    c = oracle.gemm_bf16_f64(a_bits, eye_bits)
    assert np.array_equal(c, a)
    base = oracle.gemm_bf16_f64(a_bits, b_bits)
    rng = np.random.default_rng(3)
    pm, pn, pk = rng.permutation(M), rng.permutation(N), rng.permutation(K)
    assert np.array_equal(oracle.gemm_bf16_f64(a_bits[pm], b_bits), base[pm])
    assert np.array_equal(oracle.gemm_bf16_f64(a_bits, b_bits[pn]), base[:, pn])
    assert np.array_equal(oracle.gemm_bf16_f64(a_bits[:, pk], b_bits[:, pk]), base)
    # a non-square, non-symmetric case distinguishes A.B from A.B^T / B.A
    a2, b2 = synth.bf16_operands(3, 5, 4, "ints", workload=6)
    c2 = oracle.gemm_bf16_f64(a2, b2)
    A = oracle.decode_bf16(a2)
    B_kn = oracle.decode_bf16(b2).T
    for i in range(3):
        for j in range(5):
            assert c2[i, j] == sum(A[i, k] * B_kn[k, j] for k in range(4))


def test_closed_forms():
    for K in (1, 7, 64, 256, 257, 1000):
        ones_a = synth.to_bf16_bits(np.ones((3, K)))
        ones_b = synth.to_bf16_bits(np.ones((5, K)))
        assert np.all(oracle.gemm_bf16_f64(ones_a, ones_b) == K)
    for K in (1, 2, 10, 100, 257):                  # k <= 256 is exact in bf16
        ramp = synth.to_bf16_bits(np.tile(np.arange(K, dtype=np.float64), (4, 1)))
        ones_b = synth.to_bf16_bits(np.ones((6, K)))
        assert np.all(oracle.gemm_bf16_f64(ramp, ones_b) == K * (K - 1) // 2)
    # signs: (-A).B = -(A.B); sum|ab| ignores the signs
    a_bits, b_bits = synth.bf16_operands(9, 11, 30, "normal", workload=8)
    c, s = oracle.gemm_bf16_f64(a_bits, b_bits, with_abs=True)
    neg = a_bits ^ np.uint16(0x8000)
    c2, s2 = oracle.gemm_bf16_f64(neg, b_bits, with_abs=True)
    assert np.array_equal(c2, -c) and np.array_equal(s2, s)
    assert np.all(s >= np.abs(c))


def test_empty_and_zero_k():
    a = np.zeros((4, 0), np.uint16)
    b = np.zeros((3, 0), np.uint16)
    assert np.array_equal(oracle.gemm_bf16_f64(a, b), np.zeros((4, 3)))
    assert oracle.gemm_bf16_f64(np.zeros((0, 5), np.uint16), np.zeros((3, 5), np.uint16)).shape == (0, 3)


def test_nan_propagates_to_row_and_column():
    a_bits, b_bits = synth.bf16_operands(6, 7, 8, "uniform", workload=9)
    a_bits = a_bits.copy()
    b_bits = b_bits.copy()
    a_bits[2, 5] = 0x7FC0
    b_bits[4, 1] = 0x7FC0
    c = oracle.gemm_bf16_f64(a_bits, b_bits)
    nan = np.isnan(c)
    assert nan[2, :].all() and nan[:, 4].all()
    assert nan.sum() == 7 + 6 - 1


def test_sampled_subblock_equals_full():
    a_bits, b_bits = synth.bf16_operands(70, 50, 40, "normal", workload=10, lda=48, ldb=40)
    full = oracle.gemm_bf16_f64(a_bits, b_bits, K=40)
    rows = np.array([0, 13, 69])
    cols = np.array([49, 0, 7, 31])
    sub = oracle.gemm_bf16_f64(a_bits, b_bits, K=40, rows=rows, cols=cols)
    assert np.array_equal(sub, full[np.ix_(rows, cols)])


def test_cross_check_torch_float64_matmul():
    """Secondary check, never the oracle: torch CPU fp64 matmul."""
    a_bits, b_bits = synth.bf16_operands(65, 47, 129, "normal", workload=11)
    a = oracle.decode_bf16(a_bits)
    b = oracle.decode_bf16(b_bits)
    c, s = oracle.gemm_bf16_f64(a_bits, b_bits, with_abs=True)
    ref = (torch.from_numpy(a) @ torch.from_numpy(b).T).numpy()
    assert np.all(np.abs(c - ref) <= 1e-13 * s + 1e-300)


# ----------------------------------------------------------------- MXFP8 --

def test_mxfp8_unit_scales_reduce_to_plain_gemm():
    a, sfa, b, sfb = synth.mxfp8_operands(20, 24, 96, workload=12)
    sfa[:] = 127
    sfb[:] = 127
    c = oracle.gemm_mxfp8_f64(a, sfa, b, sfb)
    want = oracle.gemm_f64(oracle.decode_e4m3(a), oracle.decode_e4m3(b))
    assert np.array_equal(c, want)


def test_mxfp8_scale_block_pins():
    """Raising one block's scale byte by one doubles exactly that block's
    contribution (integer-valued elements keep every sum exact)."""
    M, N, K = 6, 5, 128
    ints_a = synth.small_ints(1, (M, K))
    ints_b = synth.small_ints(2, (N, K))
    a = synth.to_e4m3_codes(ints_a)
    b = synth.to_e4m3_codes(ints_b)
    sfa = np.full((M, K // 32), 127, np.uint8)
    sfb = np.full((N, K // 32), 127, np.uint8)
    base = oracle.gemm_mxfp8_f64(a, sfa, b, sfb)
    i, blk = 3, 2
    sfa2 = sfa.copy()
    sfa2[i, blk] = 128
    c2 = oracle.gemm_mxfp8_f64(a, sfa2, b, sfb)
    ks = slice(32 * blk, 32 * blk + 32)
    block = ints_a[i, ks] @ ints_b[:, ks].T
    assert np.array_equal(c2[i] - base[i], block)
    others = [r for r in range(M) if r != i]
    assert np.array_equal(c2[others], base[others])
    # a B-side scale acts on a column, and scales multiply: 2^(sa-127) 2^(sb-127)
    sfb2 = sfb.copy()
    sfb2[1, 0] = 125
    c3 = oracle.gemm_mxfp8_f64(a, sfa, b, sfb2)
    block0 = ints_a[:, :32] @ ints_b[1, :32]
    assert np.array_equal(c3[:, 1] - base[:, 1], block0 * (0.25 - 1.0))
    # decode of a scaled operand
    vals = oracle.decode_mx_operand(a, sfa2, K)
    assert np.array_equal(vals[i, ks], 2.0 * ints_a[i, ks])
    assert np.array_equal(vals[i, :32], ints_a[i, :32])


def test_mxfp8_brute_force_tiny():
    for K in (32, 64):
        a, sfa, b, sfb = synth.mxfp8_operands(3, 4, K, workload=13 + K)
        c = oracle.gemm_mxfp8_f64(a, sfa, b, sfb)
        av = oracle.decode_e4m3(a)
        bv = oracle.decode_e4m3(b)
        for i in range(3):
            for j in range(4):
                want = Fraction(0)
                for k in range(K):
                    sa = Fraction(2) ** (int(sfa[i, k // 32]) - 127)
                    sb = Fraction(2) ** (int(sfb[j, k // 32]) - 127)
                    want += Fraction(float(av[i, k])) * sa * Fraction(float(bv[j, k])) * sb
                assert Fraction(c[i, j]) == want


def test_line_sums_match_full_product():
    """The row/column-sum identity used for full-size checks agrees with the
    full oracle product (exactly, on integers)."""
    a_bits, b_bits = synth.bf16_operands(37, 29, 70, "ints", workload=14)
    a = oracle.decode_bf16(a_bits)
    b = oracle.decode_bf16(b_bits)
    c, s = oracle.gemm_bf16_f64(a_bits, b_bits, with_abs=True)
    rows, rows_mag, cols, cols_mag = oracle.gemm_line_sums_f64(a, b)
    assert np.array_equal(rows, c.sum(axis=1)) and np.array_equal(cols, c.sum(axis=0))
    assert np.array_equal(rows_mag, s.sum(axis=1)) and np.array_equal(cols_mag, s.sum(axis=0))


def test_axpby_epilogue_closed_forms():
    ab = np.array([[1.0, -2.0], [3.5, 0.25]])
    old = np.array([[10.0, np.nan], [-4.0, 8.0]])
    assert np.array_equal(oracle.axpby(ab, old, 1.0, 0.0), ab)            # beta = 0: old C ignored, NaN too
    got = oracle.axpby(ab, np.nan_to_num(old), 2.0, -1.0)
    assert np.array_equal(got, np.array([[2.0 - 10.0, -4.0], [7.0 + 4.0, 0.5 - 8.0]]))
    assert np.array_equal(oracle.axpby(np.zeros((2, 2)), np.nan_to_num(old), 3.0, 0.5), 0.5 * np.nan_to_num(old))


def test_gelu_relu_closed_forms():
    # Phi(1) and Phi(-1) from the standard normal table; GELU(x) = x Phi(x)
    assert oracle.gelu(np.array([1.0]))[0] == pytest.approx(0.8413447460685429, abs=1e-15)
    assert oracle.gelu(np.array([-1.0]))[0] == pytest.approx(-0.15865525393145707, abs=1e-15)
    assert oracle.gelu(np.array([0.0]))[0] == 0.0
    x = np.linspace(-6.0, 6.0, 121)
    # Phi(x) + Phi(-x) = 1, so GELU(x) - GELU(-x) = x
    assert np.allclose(oracle.gelu(x) - oracle.gelu(-x), x, atol=1e-15, rtol=0)
    assert np.allclose(oracle.gelu(np.array([40.0, -40.0])), [40.0, 0.0], atol=1e-300)
    r = oracle.relu(np.array([-2.0, -0.0, 0.0, 3.5, np.nan]))
    assert np.array_equal(r[:4], [0.0, 0.0, 0.0, 3.5]) and np.isnan(r[4])


def test_epilogue_order_and_bias_broadcast():
    ab = np.array([[1.0, -2.0, 0.5], [3.0, 0.0, -1.0]])
    old = np.array([[1.0, 1.0, 1.0], [2.0, 2.0, 2.0]])
    bias = np.array([0.0, 10.0, -1.0])
    lin = oracle.epilogue(ab, old, 2.0, -1.0, bias, oracle.ACT_NONE)
    assert np.array_equal(lin, np.array([[1.0, 5.0, -1.0], [4.0, 8.0, -5.0]]))
    # the activation comes last: relu after bias, not before
    assert np.array_equal(oracle.epilogue(ab, old, 2.0, -1.0, bias, oracle.ACT_RELU),
                          np.array([[1.0, 5.0, 0.0], [4.0, 8.0, 0.0]]))
    assert np.allclose(oracle.epilogue(ab, old, 2.0, -1.0, bias, oracle.ACT_GELU), oracle.gelu(lin))
    assert np.array_equal(oracle.epilogue(ab, old, 1.0, 0.0, None, oracle.ACT_NONE), ab)
    with pytest.raises(ValueError):
        oracle.epilogue(ab, old, 1.0, 0.0, None, 7)


def test_fusion_saving_is_one_write_and_one_read():
    # an 8192 x 8192 fp32 intermediate: 268 MB out and 268 MB back in
    assert oracle.fusion_saving_bytes(8192 * 8192 * 4) == 536870912


def test_gelu_tanh_form_closed_forms():
    # tanh is odd, so the tanh form keeps GELU(x) - GELU(-x) = x
    x = np.linspace(-6.0, 6.0, 121)
    assert np.allclose(oracle.gelu_tanh(x) - oracle.gelu_tanh(-x), x, atol=1e-15, rtol=0)
    # at x = 1: 0.5 (1 + tanh(sqrt(2/pi) * 1.044715))
    assert oracle.gelu_tanh(np.array([1.0]))[0] == pytest.approx(0.8411919906082768, abs=1e-15)
    # it tracks the erf form to within 4.8e-4, the largest gap (about 4.73e-4)
    # lying near x = 2.7; a wrong cubic coefficient moves both
    xs = np.linspace(-10.0, 10.0, 200001)
    gap = np.abs(oracle.gelu_tanh(xs) - oracle.gelu(xs))
    assert 4.6e-4 < gap.max() < 4.8e-4
    assert 2.5 < abs(xs[gap.argmax()]) < 2.9
    assert np.array_equal(oracle.epilogue(np.array([[1.0]]), None, 1.0, 0.0, None, oracle.ACT_GELU_TANH),
                          oracle.gelu_tanh(np.array([[1.0]])))
