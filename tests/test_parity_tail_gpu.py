"""GPU parity of the narrow tail: when the tiles left for a last wave would
occupy at most half of the co-resident clusters, each of them runs as two
half-width units (an MMA of N = BN / 2 over half of the B rows).  Compared
with the oracle element by element; integer inputs bit-exact.

The shapes are chosen so that the tail splits for any co-resident count a
B200 gives (66-74 CTA pairs, 132-148 CTAs):
  pair tiles 256 x 256      2300 x 2500:  9 x 10 =  90 tiles (R = 16 .. 24)
  one-CTA tiles 128 x 256   2300 x 2500: 18 x 10 = 180 tiles (R = 32 .. 48)
  one-CTA tiles 128 x 128   2300 x 1250: 18 x 10 = 180 tiles
and, with no whole wave at all (every unit a half),
  pair tiles                1500 x 1250:  6 x 5  =  30 tiles
  one-CTA tiles 128 x 256   1250 x 1500: 10 x 6  =  60 tiles
A B stored K x N keeps whole tiles (the halves read B K-major); that path
must stay correct on the same shapes.
"""
import numpy as np
import pytest
import torch

import oracle
from dense_gemm_engineering_bf16_b200 import gemm as G
from dense_gemm_engineering_bf16_b200 import synth

from gpu_helpers import assert_close, assert_exact, run_gemm, to_device_bf16

pytestmark = pytest.mark.gpu
F32, BF16 = G.OUT_F32, G.OUT_BF16

CASES = [("2cta_256x256", 2300, 2500), ("2cta_256x256_clc", 2300, 2500), ("1cta_128x256", 2300, 2500),
         ("1cta_128x256_clc", 2300, 2500), ("1cta_128x128", 2300, 1250), ("2cta_256x256", 1500, 1250),
         ("2cta_256x256_clc", 1500, 1250), ("1cta_128x256", 1250, 1500)]
IDS = [f"{c}-{m}x{n}" for c, m, n in CASES]


@pytest.mark.parametrize("c_type", [F32, BF16])
@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_integers_bit_exact(case, c_type):
    cfg, M, N = case
    K = 328
    a_bits, b_bits = synth.bf16_operands(M, N, K, "ints", workload=600 + M % 7)
    got, guard_ok = run_gemm(a_bits, b_bits, M, N, K, c_type=c_type, config=cfg).download()
    assert guard_ok, "write outside C's M x N window"
    assert_exact(got, oracle.gemm_bf16_f64(a_bits, b_bits, K=K), c_type, f"{cfg} {M}x{N}x{K}")


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_normal_within_tolerance(case):
    cfg, M, N = case
    K = 200
    a_bits, b_bits = synth.bf16_operands(M, N, K, "normal", workload=610 + N % 11)
    got, guard_ok = run_gemm(a_bits, b_bits, M, N, K, config=cfg).download()
    assert guard_ok
    c_ref, s_abs = oracle.gemm_bf16_f64(a_bits, b_bits, K=K, with_abs=True)
    assert_close(got, c_ref, s_abs, F32, f"{cfg} {M}x{N}x{K}")


@pytest.mark.parametrize("cfg", ["2cta_256x256_clc", "1cta_128x256", "1cta_128x128"])
@pytest.mark.parametrize("layouts", [(G.MNMAJOR, G.KMAJOR), (G.KMAJOR, G.MNMAJOR)], ids=["A_KxM", "B_KxN"])
def test_fused_epilogue_and_layouts(cfg, layouts):
    """alpha, beta, bias and GELU on the half units, with A stored K x M (the
    tail splits) or B stored K x N (whole tiles).  M and N are multiples of 8
    here: a transposed operand's rows must start on 16-byte boundaries."""
    M, N, K = (2296, 1256, 264) if cfg == "1cta_128x128" else (2296, 2504, 264)
    a_lay, b_lay = layouts
    a_bits, b_bits = synth.bf16_operands(M, N, K, "normal", workload=620)
    a_dev = np.ascontiguousarray(a_bits.T) if a_lay == G.MNMAJOR else a_bits
    b_dev = np.ascontiguousarray(b_bits.T) if b_lay == G.MNMAJOR else b_bits
    lda = M if a_lay == G.MNMAJOR else K
    ldb = N if b_lay == G.MNMAJOR else K
    c_old = synth.normal(621, (M, N)).astype(np.float32)
    bias = synth.uniform(622, (N,)).astype(np.float32)
    C = torch.from_numpy(c_old).cuda()
    G.gemm_force_config(cfg)
    try:
        G.gemm_bf16_fused(to_device_bf16(a_dev), to_device_bf16(b_dev), C, M, N, K, lda, ldb, N, F32, a_lay, b_lay,
                          0.75, -0.5, torch.from_numpy(bias).cuda(), G.ACT_GELU)
    finally:
        G.gemm_force_config("auto")
    G.gemm_check_device_status()
    got = C.cpu().numpy().astype(np.float64)
    ab, s = oracle.gemm_bf16_f64(a_bits, b_bits, with_abs=True)
    old = c_old.astype(np.float64)
    want = oracle.epilogue(ab, old, 0.75, -0.5, bias.astype(np.float64), G.ACT_GELU)
    lin = oracle.axpby(ab, old, 0.75, -0.5) + bias.astype(np.float64)[None, :]
    # the GEMM's tolerance through alpha, the rounding of beta C, then GELU's
    # slope (at most 1.13) and the fp32 evaluation of the activation
    tol = 1.13 * (0.75 * (1e-3 * s + 1e-6) + 1e-6 * np.abs(0.5 * old)) + 1e-6 * np.abs(lin) + 1e-6
    bad = np.abs(got - want) > tol
    assert not bad.any(), f"{cfg} {layouts}: {int(bad.sum())} elements off, first at {np.argwhere(bad)[0]}"
