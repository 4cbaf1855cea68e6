"""GPU parity of gemm_bf16_ex: C = alpha A.B + beta C with K-major or
MN-major operands (A stored M x K or K x M, B stored N x K or K x N), in
every kernel configuration, against the oracle on the canonical operands."""
import numpy as np
import pytest
import torch

import oracle
from dense_gemm_engineering_bf16_b200 import gemm as G
from dense_gemm_engineering_bf16_b200 import synth

from gpu_helpers import assert_close, assert_exact, sample_indices, to_device_bf16

pytestmark = pytest.mark.gpu
F32, BF16 = G.OUT_F32, G.OUT_BF16
K_, MN = G.KMAJOR, G.MNMAJOR
CFGS = ["1cta_128x128", "1cta_128x256", "2cta_256x256", "2cta_256x256_clc", "2cta_512x256_clc", "skinny",
        "2cta_256x256_sk", "2cta_256x224", "1cta_128x128_splitk", "1cta_128x256_splitk"]


def _store(canon_bits: np.ndarray, mn: bool) -> np.ndarray:
    """Canonical operand (rows x K) -> stored array: as is (K-major), or
    transposed to K x rows with the row pitch padded to 8 elements."""
    if not mn:
        return canon_bits
    t = np.ascontiguousarray(canon_bits.T)
    pad = -t.shape[1] % 8
    if pad:
        t = np.concatenate([t, np.full((t.shape[0], pad), 0x7FC0, np.uint16)], axis=1)
    return t


def _run(M, N, K, dist, workload, cfg, a_layout, b_layout, alpha=1.0, beta=0.0, c_type=F32, c_old=None):
    a_bits, b_bits = synth.bf16_operands(M, N, K, dist, workload=workload)
    A_st, B_st = _store(a_bits, a_layout == MN), _store(b_bits, b_layout == MN)
    ldc = N + (-N % 8)
    if c_old is None:
        c_old = np.zeros((M, N))
    dt = torch.float32 if c_type == F32 else torch.bfloat16
    C = torch.full((M, ldc), float("nan"), dtype=dt)
    C[:, :N] = torch.from_numpy(c_old).to(dt)
    C = C.cuda()
    G.gemm_force_config(cfg)
    try:
        G.gemm_bf16_ex(to_device_bf16(A_st), to_device_bf16(B_st), C, M, N, K, A_st.shape[1], B_st.shape[1], ldc,
                       c_type, a_layout, b_layout, alpha, beta)
    finally:
        G.gemm_force_config("auto")
    G.gemm_check_device_status()
    host = C.cpu()
    got = host.float().numpy().astype(np.float64)
    assert np.isnan(got[:, N:]).all(), "wrote past column N"
    c_ab, s_abs = oracle.gemm_bf16_f64(a_bits, b_bits, with_abs=True)
    old_used = torch.from_numpy(c_old).to(dt).float().numpy().astype(np.float64)   # C as stored
    want = oracle.axpby(c_ab, old_used, alpha, beta)
    return got[:, :N], want, s_abs, old_used


@pytest.mark.parametrize("cfg", CFGS)
@pytest.mark.parametrize("layouts", [(K_, MN), (MN, K_), (MN, MN)], ids=["B_KxN", "A_KxM", "both_MN"])
@pytest.mark.parametrize("shape", [(300, 200, 136), (129, 257, 200), (256, 512, 1024)],
                         ids=lambda s: "x".join(map(str, s)))
def test_operand_layouts_integers_bit_exact(cfg, layouts, shape):
    a_l, b_l = layouts
    M, N, K = shape
    if cfg == "skinny":                  # the swap-AB path takes at most 256 rows; with A stored
        M = min(M, 250)                  # K x M the call is routed to the 128 x 128 split-K kernel
    got, want, _, _ = _run(M, N, K, "ints", 200 + M, cfg, a_l, b_l)
    assert_exact(got, want, F32, f"{cfg} layouts {layouts} {shape}")


@pytest.mark.parametrize("cfg", CFGS)
@pytest.mark.parametrize("c_type", [F32, BF16])
def test_alpha_beta_integers_bit_exact(cfg, c_type):
    M, N, K = 200, 300, 512
    c_old = synth.small_ints(7, (M, N), -8, 8)
    got, want, _, _ = _run(M, N, K, "ints", 210, cfg, K_, MN if cfg != "skinny" else K_,
                           alpha=2.0, beta=-1.0, c_type=c_type, c_old=c_old)
    assert_exact(got, want, c_type, f"{cfg} alpha/beta")


@pytest.mark.parametrize("cfg", CFGS)
@pytest.mark.parametrize("c_type", [F32, BF16])
def test_alpha_beta_random(cfg, c_type):
    M, N, K = (250 if cfg == "skinny" else 257), 384, 1000
    c_old = synth.normal(8, (M, N))
    alpha, beta = 0.75, 0.5
    got, want, s_abs, old = _run(M, N, K, "normal", 211, cfg, K_, K_, alpha=alpha, beta=beta,
                                 c_type=c_type, c_old=c_old)
    tol = abs(alpha) * (1e-3 * s_abs + 1e-6) + 1e-6 * np.abs(beta * old) + 1e-6
    if c_type == BF16:
        tol = tol + 2.0 ** -8 * np.abs(want)
    assert np.all(np.abs(got - want) <= tol)


def test_beta_zero_ignores_nan_in_c():
    M, N, K = 130, 140, 256
    c_old = np.full((M, N), np.nan)
    got, want, s_abs, _ = _run(M, N, K, "normal", 212, "1cta_128x128", K_, K_, alpha=1.5, beta=0.0, c_old=c_old)
    assert np.isfinite(got).all()
    assert np.all(np.abs(got - want) <= 1.5 * (1e-3 * s_abs + 1e-6))


@pytest.mark.parametrize("beta", [0.0, -2.5])
def test_k_zero_is_beta_times_c(beta):
    M, N = 70, 92
    c_old = synth.normal(9, (M, N))
    C = torch.from_numpy(c_old.astype(np.float32)).cuda()
    A = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    G.gemm_bf16_ex(A, A, C, M, N, 0, 8, 8, N, F32, K_, K_, 3.0, beta)
    G.gemm_check_device_status()
    got = C.cpu().numpy().astype(np.float64)
    assert np.array_equal(got, (np.float32(beta) * c_old.astype(np.float32)).astype(np.float64))


def test_layouts_at_4096_cube_against_k_major():
    """A stored K x M and B stored K x N (torch's own layout for A @ B) at
    4096^3 on the shape-chosen kernel: identical to the K-major result."""
    M = N = K = 4096
    a_bits, b_bits = synth.bf16_operands(M, N, K, "normal_scaled", workload=2)
    A, B = to_device_bf16(a_bits), to_device_bf16(b_bits)
    At, Bt = to_device_bf16(np.ascontiguousarray(a_bits.T)), to_device_bf16(np.ascontiguousarray(b_bits.T))
    C1 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    C2 = torch.empty_like(C1)
    G.gemm_bf16(A, B, C1, M, N, K, K, K, N)
    G.gemm_bf16_ex(At, Bt, C2, M, N, K, M, N, N, F32, MN, MN, 1.0, 0.0)
    G.gemm_check_device_status()
    got = C2.cpu().numpy().astype(np.float64)
    rows = sample_indices(M, 128, 24, seed=5)
    cols = sample_indices(N, 128, 24, seed=6)
    c_ref, s_abs = oracle.gemm_bf16_f64(a_bits, b_bits, rows=rows, cols=cols, with_abs=True)
    assert_close(got[np.ix_(rows, cols)], c_ref, s_abs, F32, "4096^3 K x M / K x N")
    # the tensor core sums the same products whichever way the tiles sit in shared memory
    assert torch.equal(C1, C2)
