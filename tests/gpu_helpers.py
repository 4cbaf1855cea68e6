"""Shared helpers for the GPU parity tests: upload seeded operands, run the
library through its C ABI with guard bands around C, and compare with the
oracle under the stated tolerance.

Tolerance (per element, fp32 output):  |C - C_ref| <= 1e-3 * S + 1e-6,
S = sum_k |a_ik b_kj|.  bf16 output adds half a bf16 ulp of the result,
2^-8 |C_ref|, for the final rounding.  Integer-valued inputs must match
bit for bit.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from dense_gemm_engineering_bf16_b200 import gemm as G

GUARD_ROWS = 3
SENTINEL_F32 = np.uint32(0x7FC0DEAD)   # a NaN payload no kernel writes
SENTINEL_BF16 = np.uint16(0x7FAB)


def to_device_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


class GuardedC:
    """C storage of (M + 2*GUARD_ROWS) x ldc elements filled with a sentinel;
    the kernel sees rows GUARD_ROWS .. GUARD_ROWS+M-1, columns 0..N-1."""

    def __init__(self, M: int, N: int, ldc: int, c_type: int):
        self.M, self.N, self.ldc, self.c_type = M, N, ldc, c_type
        rows = M + 2 * GUARD_ROWS
        if c_type == G.OUT_F32:
            host = np.full(rows * ldc, SENTINEL_F32, dtype=np.uint32).view(np.int32)
            self.raw = torch.from_numpy(host).cuda()
            self.esize = 4
        else:
            host = np.full(rows * ldc, SENTINEL_BF16, dtype=np.uint16).view(np.int16)
            self.raw = torch.from_numpy(host).cuda()
            self.esize = 2
        self.ptr = self.raw.data_ptr() + GUARD_ROWS * ldc * self.esize

    def download(self):
        """(values as fp64 M x N, guard-intact flag)."""
        rows = self.M + 2 * GUARD_ROWS
        if self.c_type == G.OUT_F32:
            host = self.raw.cpu().numpy().view(np.uint32).reshape(rows, self.ldc)
            sentinel = SENTINEL_F32
            body = host[GUARD_ROWS:GUARD_ROWS + self.M, :self.N].view(np.float32).astype(np.float64)
        else:
            host = self.raw.cpu().numpy().view(np.uint16).reshape(rows, self.ldc)
            sentinel = SENTINEL_BF16
            body = oracle.decode_bf16(host[GUARD_ROWS:GUARD_ROWS + self.M, :self.N])
        guard_ok = bool(np.all(host[:GUARD_ROWS] == sentinel) and np.all(host[GUARD_ROWS + self.M:] == sentinel)
                        and np.all(host[GUARD_ROWS:GUARD_ROWS + self.M, self.N:] == sentinel))
        return body, guard_ok

    def bits(self) -> np.ndarray:
        rows = self.M + 2 * GUARD_ROWS
        dt = np.uint32 if self.c_type == G.OUT_F32 else np.uint16
        host = self.raw.cpu().numpy().view(dt).reshape(rows, self.ldc)
        return host[GUARD_ROWS:GUARD_ROWS + self.M, :self.N].copy()


def run_gemm(a_bits: np.ndarray, b_bits: np.ndarray, M: int, N: int, K: int,
             c_type: int = G.OUT_F32, ldc: int | None = None, config: str = "auto",
             repeats: int = 1):
    """Run C = A.B on the GPU through the C ABI; returns the GuardedC."""
    lda = a_bits.shape[1] if a_bits.ndim == 2 and a_bits.shape[0] else max(K, 8)
    ldb = b_bits.shape[1] if b_bits.ndim == 2 and b_bits.shape[0] else max(K, 8)
    if ldc is None:
        ldc = N + (-N % (4 if c_type == G.OUT_F32 else 8))
    A = to_device_bf16(a_bits) if a_bits.size else torch.empty(16, dtype=torch.bfloat16, device="cuda")
    B = to_device_bf16(b_bits) if b_bits.size else torch.empty(16, dtype=torch.bfloat16, device="cuda")
    C = GuardedC(M, N, ldc, c_type)
    G.gemm_force_config(config)
    try:
        for _ in range(repeats):
            G.gemm_bf16(A, B, C.ptr, M, N, K, lda, ldb, ldc, c_type)
    finally:
        G.gemm_force_config("auto")
    G.gemm_check_device_status()
    torch.cuda.synchronize()
    return C


def tolerance(c_ref: np.ndarray, s_abs: np.ndarray, c_type: int) -> np.ndarray:
    tol = 1e-3 * s_abs + 1e-6
    if c_type == G.OUT_BF16:
        tol = tol + np.abs(c_ref) * 2.0 ** -8
    return tol


def assert_close(got: np.ndarray, c_ref: np.ndarray, s_abs: np.ndarray, c_type: int, what: str = ""):
    tol = tolerance(c_ref, s_abs, c_type)
    nan_ref = np.isnan(c_ref)
    assert np.array_equal(np.isnan(got), nan_ref), f"{what}: NaN pattern differs"
    err = np.abs(got - c_ref)
    bad = (err > tol) & ~nan_ref
    if bad.any():
        idx = np.argwhere(bad)[:5]
        detail = ", ".join(f"({i},{j}) got {got[i, j]!r} want {c_ref[i, j]!r} tol {tol[i, j]:.3g}" for i, j in idx)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} elements outside tolerance: {detail}")


def assert_exact(got: np.ndarray, c_ref: np.ndarray, c_type: int, what: str = ""):
    """Bit-exact comparison against the oracle's single final rounding."""
    want = oracle.round_f32(c_ref).astype(np.float64) if c_type == G.OUT_F32 else \
        oracle.decode_bf16(oracle.round_bf16(c_ref))
    bad = got != want
    if bad.any():
        idx = np.argwhere(bad)[:5]
        detail = ", ".join(f"({i},{j}) got {got[i, j]!r} want {want[i, j]!r}" for i, j in idx)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} elements differ: {detail}")


def sample_indices(n: int, tile: int, extra: int, seed: int) -> np.ndarray:
    """Indices touching every tile boundary (first / last row of a tile) plus
    random ones, sorted and unique."""
    idx = set()
    for t in range(0, n, tile):
        idx.update({t, min(n - 1, t + tile - 1)})
    idx.update({0, n - 1})
    idx = sorted(idx)
    if len(idx) > 48:
        rng = np.random.default_rng(seed)
        idx = sorted(rng.choice(idx, 48, replace=False).tolist() + [0, n - 1])
    rng = np.random.default_rng(seed + 1)
    extra_idx = rng.integers(0, n, size=extra).tolist()
    return np.array(sorted(set(idx) | set(extra_idx)), dtype=np.int64)


def run_mxfp8(a_codes: np.ndarray, sfa: np.ndarray, b_codes: np.ndarray, sfb: np.ndarray,
              M: int, N: int, K: int, ldc: int | None = None, config: str = "auto"):
    """Run the block-scaled GEMM through the C ABI; returns the GuardedC (bf16)."""
    lda = a_codes.shape[1] if a_codes.size else 16
    ldb = b_codes.shape[1] if b_codes.size else 16
    if ldc is None:
        ldc = N + (-N % 8)

    def dev(x):
        x = np.ascontiguousarray(x, dtype=np.uint8)
        return torch.from_numpy(x).cuda() if x.size else torch.empty(16, dtype=torch.uint8, device="cuda")

    A, B, SA, SB = dev(a_codes), dev(b_codes), dev(sfa), dev(sfb)
    C = GuardedC(M, N, ldc, G.OUT_BF16)
    G.gemm_force_config(config)
    try:
        G.gemm_mxfp8(A, SA, B, SB, C.ptr, M, N, K, lda, ldb, ldc)
    finally:
        G.gemm_force_config("auto")
    G.gemm_check_device_status()
    torch.cuda.synchronize()
    return C
