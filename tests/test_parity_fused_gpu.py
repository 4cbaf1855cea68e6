"""GPU parity of gemm_bf16_fused: C = act(alpha A.B + beta C + bias) with the
bias and the activation applied in the GEMM's write-back, in every kernel
configuration, against the oracle's fp64 epilogue."""
import numpy as np
import pytest
import torch

import oracle
from dense_gemm_engineering_bf16_b200 import gemm as G
from dense_gemm_engineering_bf16_b200 import synth

from gpu_helpers import assert_exact, to_device_bf16

pytestmark = pytest.mark.gpu
F32, BF16 = G.OUT_F32, G.OUT_BF16
CFGS = ["1cta_128x128", "1cta_128x256", "2cta_256x256", "2cta_256x256_clc", "2cta_512x256_clc", "skinny",
        "2cta_256x256_sk", "2cta_256x224", "1cta_128x128_splitk", "1cta_128x256_splitk"]
ACTS = {"none": G.ACT_NONE, "relu": G.ACT_RELU, "gelu": G.ACT_GELU, "gelu_tanh": G.ACT_GELU_TANH}


def _run(M, N, K, dist, workload, cfg, act, alpha=1.0, beta=0.0, c_type=F32, c_old=None, bias=None,
         b_layout=G.KMAJOR):
    a_bits, b_bits = synth.bf16_operands(M, N, K, dist, workload=workload)
    B_st = b_bits if b_layout == G.KMAJOR else np.ascontiguousarray(b_bits.T)
    ldc = N + (-N % 8)
    if c_old is None:
        c_old = np.zeros((M, N))
    dt = torch.float32 if c_type == F32 else torch.bfloat16
    C = torch.full((M, ldc), float("nan"), dtype=dt)
    C[:, :N] = torch.from_numpy(c_old).to(dt)
    C = C.cuda()
    bias_d = None if bias is None else torch.from_numpy(bias.astype(np.float32)).cuda()
    G.gemm_force_config(cfg)
    try:
        G.gemm_bf16_fused(to_device_bf16(a_bits), to_device_bf16(B_st), C, M, N, K, K, B_st.shape[1], ldc,
                          c_type, G.KMAJOR, b_layout, alpha, beta, bias_d, act)
    finally:
        G.gemm_force_config("auto")
    G.gemm_check_device_status()
    got = C.cpu().float().numpy().astype(np.float64)
    assert np.isnan(got[:, N:]).all(), "wrote past column N"
    c_ab, s_abs = oracle.gemm_bf16_f64(a_bits, b_bits, with_abs=True)
    old_used = torch.from_numpy(c_old).to(dt).float().numpy().astype(np.float64)
    bias64 = None if bias is None else bias.astype(np.float32).astype(np.float64)
    want = oracle.epilogue(c_ab, old_used, alpha, beta, bias64, act)
    lin = oracle.axpby(c_ab, old_used, alpha, beta) + (0.0 if bias64 is None else bias64[None, :])
    return got[:, :N], want, s_abs, old_used, lin


def _tolerance(want, s_abs, old, lin, alpha, beta, c_type, act):
    t = abs(alpha) * (1e-3 * s_abs + 1e-6) + 1e-6 * np.abs(beta * old)
    if act == G.ACT_GELU:
        # |GELU'| <= 1.13; fp32 erff and the products add a few ulp of |x|
        t = 1.13 * t + 1e-6 * np.abs(lin) + 1e-6
    if act == G.ACT_GELU_TANH:
        # the same slope bound; the hardware tanh is within 2^-10 of tanh,
        # which 0.5 x scales to 2^-11 |x|
        t = 1.13 * t + 2.0 ** -11 * np.abs(lin) + 1e-6
    if c_type == BF16:
        t = t + 2.0 ** -8 * np.abs(want)
    return t


@pytest.mark.parametrize("cfg", CFGS)
@pytest.mark.parametrize("act", ["relu", "gelu", "gelu_tanh"])
@pytest.mark.parametrize("c_type", [F32, BF16])
def test_bias_activation_random(cfg, act, c_type):
    M, N, K = (250 if cfg == "skinny" else 257), 300, 1000
    bias = synth.normal(31, (N,))
    got, want, s_abs, old, lin = _run(M, N, K, "normal", 300, cfg, ACTS[act], c_type=c_type, bias=bias)
    tol = _tolerance(want, s_abs, old, lin, 1.0, 0.0, c_type, ACTS[act])
    bad = np.abs(got - want) > tol
    assert not bad.any(), f"{int(bad.sum())} elements out of tolerance"
    if act == "relu":
        assert (got >= 0).all()


@pytest.mark.parametrize("cfg", CFGS)
def test_alpha_beta_bias_gelu_with_transposed_b(cfg):
    M, N, K = (200 if cfg == "skinny" else 300), 264, 704
    c_old = synth.normal(32, (M, N))
    bias = synth.uniform(33, (N,))
    got, want, s_abs, old, lin = _run(M, N, K, "normal", 301, cfg, G.ACT_GELU, alpha=0.5, beta=-1.5,
                                      c_old=c_old, bias=bias, b_layout=G.MNMAJOR)
    tol = _tolerance(want, s_abs, old, lin, 0.5, -1.5, F32, G.ACT_GELU)
    assert np.all(np.abs(got - want) <= tol)


@pytest.mark.parametrize("cfg", CFGS)
@pytest.mark.parametrize("c_type", [F32, BF16])
def test_integer_bias_relu_bit_exact(cfg, c_type):
    M, N, K = (129 if cfg == "skinny" else 200), 140, 512
    c_old = synth.small_ints(34, (M, N), -8, 8)
    bias = synth.small_ints(35, (N,), -20, 20)
    got, want, _, _, _ = _run(M, N, K, "ints", 302, cfg, G.ACT_RELU, alpha=1.0, beta=-1.0, c_type=c_type,
                              c_old=c_old, bias=bias)
    assert_exact(got, want, c_type, f"{cfg} ints bias relu")


@pytest.mark.parametrize("act", ["none", "relu", "gelu", "gelu_tanh"])
def test_k_zero_is_epilogue_of_zero(act):
    M, N = 40, 72
    c_old = synth.normal(36, (M, N)).astype(np.float32)
    bias = synth.normal(37, (N,)).astype(np.float32)
    C = torch.from_numpy(c_old.copy()).cuda()
    A = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    G.gemm_bf16_fused(A, A, C, M, N, 0, 8, 8, N, F32, G.KMAJOR, G.KMAJOR, 2.0, 0.5,
                      torch.from_numpy(bias).cuda(), ACTS[act])
    G.gemm_check_device_status()
    got = C.cpu().numpy().astype(np.float64)
    want = oracle.epilogue(np.zeros((M, N)), c_old.astype(np.float64), 2.0, 0.5, bias.astype(np.float64), ACTS[act])
    lin = 0.5 * c_old.astype(np.float64) + bias.astype(np.float64)[None, :]
    tol = 1e-6 * np.abs(want) + 1e-6 + (2.0 ** -11 * np.abs(lin) if act == "gelu_tanh" else 0.0)
    assert np.all(np.abs(got - want) <= tol)


def test_activation_without_bias_and_identity_matches_plain():
    M, N, K = 256, 256, 512
    a_bits, b_bits = synth.bf16_operands(M, N, K, "uniform", workload=303)
    A, B = to_device_bf16(a_bits), to_device_bf16(b_bits)
    C1 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    C2 = torch.empty_like(C1)
    C3 = torch.empty_like(C1)
    G.gemm_bf16(A, B, C1, M, N, K, K, K, N)
    G.gemm_bf16_fused(A, B, C2, M, N, K, K, K, N, F32, G.KMAJOR, G.KMAJOR, 1.0, 0.0, None, G.ACT_NONE)
    G.gemm_bf16_fused(A, B, C3, M, N, K, K, K, N, F32, G.KMAJOR, G.KMAJOR, 1.0, 0.0, None, G.ACT_RELU)
    G.gemm_check_device_status()
    assert torch.equal(C1, C2)
    assert torch.equal(C3, torch.where(C1 < 0, torch.zeros_like(C1), C1))


def test_fused_at_8192_cube_sampled():
    """The headline shape with bias + GELU, bf16 out, on the shape-chosen kernel."""
    M = N = K = 8192
    a_bits, b_bits = synth.bf16_operands(M, N, K, "uniform", workload=3)
    bias = synth.normal(38, (N,)).astype(np.float32)
    C = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    G.gemm_bf16_fused(to_device_bf16(a_bits), to_device_bf16(b_bits), C, M, N, K, K, K, N, BF16,
                      G.KMAJOR, G.KMAJOR, 1.0, 0.0, torch.from_numpy(bias).cuda(), G.ACT_GELU)
    G.gemm_check_device_status()
    got = C.cpu().float().numpy().astype(np.float64)
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([[0, 255, 256, M - 1], rng.integers(0, M, 20)]))
    cols = np.unique(np.concatenate([[0, 255, 256, N - 1], rng.integers(0, N, 20)]))
    c_ab, s_abs = oracle.gemm_bf16_f64(a_bits, b_bits, rows=rows, cols=cols, with_abs=True)
    lin = c_ab + bias.astype(np.float64)[cols][None, :]
    want = oracle.gelu(lin)
    tol = 1.13 * (1e-3 * s_abs + 1e-6) + 1e-6 * np.abs(lin) + 1e-6 + 2.0 ** -8 * np.abs(want)
    assert np.all(np.abs(got[np.ix_(rows, cols)] - want) <= tol)
