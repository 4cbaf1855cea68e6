"""Seeded synthetic inputs for the GEMM workloads.

This module holds no GEMM arithmetic: it only draws numbers and encodes them
into the operand formats (bf16 bit patterns, FP8 E4M3 codes, E8M0 scale
bytes).  Both the GPU tests/bench and the oracle consume its output; neither
side's arithmetic lives here.

Random stream: splitmix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014): state_i = seed + (i+1)*0x9E3779B97F4A7C15,
output = mix(state_i).  Uniforms take the top 53 bits.  Normals use the
Box-Muller transform on consecutive uniform pairs.  Each tensor of each
workload gets its own seed, derived from (workload id, tensor id, base seed).

Encoding: values are first rounded to binary32, then to the operand type with
round-to-nearest-even (torch's conversions).  The encoded bits *are* the
inputs; the oracle decodes those same bits.
"""
from __future__ import annotations

import math

import numpy as np
import torch

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def splitmix64(seed: int, n: int, offset: int = 0) -> np.ndarray:
    """Outputs offset..offset+n-1 of the splitmix64 stream started at `seed`."""
    out = np.empty(n, dtype=np.uint64)
    s = np.uint64(seed & 0xFFFFFFFFFFFFFFFF)
    with np.errstate(over="ignore"):
        for lo in range(0, n, _CHUNK):
            hi = min(n, lo + _CHUNK)
            idx = np.arange(offset + lo + 1, offset + hi + 1, dtype=np.uint64)
            out[lo:hi] = _mix(s + idx * _GOLDEN)
    return out


def derive_seed(workload: int, tensor: int, base: int = 0) -> int:
    """One 64-bit seed per (workload, tensor, base) triple."""
    with np.errstate(over="ignore"):
        z = np.uint64((base * 1_000_003 + workload * 1_009 + tensor) & 0xFFFFFFFFFFFFFFFF)
        return int(_mix(np.array([z + _GOLDEN], dtype=np.uint64))[0])


def uniform01(seed: int, n: int) -> np.ndarray:
    """n doubles uniform in [0, 1) (53-bit resolution)."""
    return (splitmix64(seed, n) >> np.uint64(11)).astype(np.float64) * (1.0 / (1 << 53))


def uniform(seed: int, shape, lo: float = -1.0, hi: float = 1.0) -> np.ndarray:
    n = int(np.prod(shape))
    return (lo + (hi - lo) * uniform01(seed, n)).reshape(shape)


def normal(seed: int, shape) -> np.ndarray:
    """Standard normal via Box-Muller on consecutive uniform pairs."""
    n = int(np.prod(shape))
    pairs = (n + 1) // 2
    out = np.empty(2 * pairs, dtype=np.float64)
    for lo in range(0, pairs, _CHUNK):
        hi = min(pairs, lo + _CHUNK)
        u = (splitmix64(seed, 2 * (hi - lo), offset=2 * lo) >> np.uint64(11)).astype(np.float64) \
            * (1.0 / (1 << 53))
        u1 = u[0::2]
        u2 = u[1::2]
        r = np.sqrt(-2.0 * np.log1p(-u1))          # 1-u1 in (0, 1]
        t = 2.0 * math.pi * u2
        out[2 * lo:2 * hi:2] = r * np.cos(t)
        out[2 * lo + 1:2 * hi:2] = r * np.sin(t)
    return out[:n].reshape(shape)


def small_ints(seed: int, shape, lo: int = -4, hi: int = 4) -> np.ndarray:
    """Integers uniform in [lo, hi], as doubles."""
    n = int(np.prod(shape))
    span = hi - lo + 1
    return (lo + np.floor(uniform01(seed, n) * span)).reshape(shape)


# ---------------------------------------------------------------- encoders --

def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp64 -> binary32 -> bf16 (RNE), returned as uint16 bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def to_e4m3_codes(x: np.ndarray) -> np.ndarray:
    """fp64 -> binary32 -> FP8 E4M3 (RNE, saturated to +-448), as uint8 codes."""
    f = np.clip(np.ascontiguousarray(x, dtype=np.float32), -448.0, 448.0)
    t = torch.from_numpy(f)
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def pad_cols(a: np.ndarray, ld: int) -> np.ndarray:
    """Place a rows x cols array into a rows x ld array (ld >= cols), padding
    the extra columns with a fixed, recognisable pattern."""
    rows, cols = a.shape
    if ld == cols:
        return np.ascontiguousarray(a)
    out = np.empty((rows, ld), dtype=a.dtype)
    out[:, :cols] = a
    # pad = bf16 / fp8 NaN patterns: a kernel that reads padding would show it
    out[:, cols:] = 0x7FC0 if a.dtype == np.uint16 else 0x7F
    return out


# ------------------------------------------------------- workload recipes --

DISTS = ("uniform", "normal", "normal_scaled", "ints")


def draw(dist: str, seed: int, shape, K: int) -> np.ndarray:
    if dist == "uniform":
        return uniform(seed, shape, -1.0, 1.0)
    if dist == "normal":
        return normal(seed, shape)
    if dist == "normal_scaled":          # N(0,1)/sqrt(K), scaled before rounding
        return normal(seed, shape) / math.sqrt(K)
    if dist == "ints":
        return small_ints(seed, shape, -4, 4)
    raise ValueError(f"unknown distribution {dist!r}; expected one of {DISTS}")


def bf16_operands(M: int, N: int, K: int, dist: str, workload: int, base: int = 0,
                  lda: int | None = None, ldb: int | None = None):
    """A (uint16 [M, lda], row-major) and B (uint16 [N, ldb], K-major) bit patterns."""
    a = to_bf16_bits(draw(dist, derive_seed(workload, 0, base), (M, K), K))
    b = to_bf16_bits(draw(dist, derive_seed(workload, 1, base), (N, K), K))
    return pad_cols(a, lda or K), pad_cols(b, ldb or K)


def mxfp8_operands(M: int, N: int, K: int, workload: int, base: int = 0,
                   exp_lo: int = -4, exp_hi: int = 4):
    """E4M3 codes for A [M,K] and B [N,K] (values U[-1,1]) and E8M0 scale bytes
    SFA [M, K/32], SFB [N, K/32] with exponents uniform in [exp_lo, exp_hi]."""
    if K % 32:
        raise ValueError("K must be a multiple of 32 for one scale per 32 elements")
    a = to_e4m3_codes(uniform(derive_seed(workload, 0, base), (M, K)))
    b = to_e4m3_codes(uniform(derive_seed(workload, 1, base), (N, K)))
    sfa = (127 + small_ints(derive_seed(workload, 2, base), (M, K // 32), exp_lo, exp_hi)).astype(np.uint8)
    sfb = (127 + small_ints(derive_seed(workload, 3, base), (N, K // 32), exp_lo, exp_hi)).astype(np.uint8)
    return a, sfa, b, sfb
