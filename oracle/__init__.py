"""Oracle for C = A.B (bf16 and block-scaled FP8 inputs) -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s cpu_baseline /
reference leg may import this package.  The GPU library never imports it, and
this package imports nothing from the GPU library.

It is a plain, slow, obviously correct CPU restatement of what the GEMM path
computes:

* ``gemm_bf16_f64``: C[i][j] = sum_k a(i,k) b(k,j) in fp64, natural k order,
  over the exact values of the bf16 inputs -- the matrix product
  C_{MxN} = A_{MxK} B_{KxN} of "GPU 执行模型", section "Tile 的容量约束".
* ``gemm_mxfp8_f64``: the same sum over block-scaled FP8 operands
  (E4M3 codes, one E8M0 scale per 32 consecutive K elements) -- the
  block-scaled MMA named in "Modern GPU Programming For MLSys - 书籍总结",
  sections 2.4 and 2.6.
* ``round_f32`` / ``round_bf16``: one final round-to-nearest-even of the fp64
  sum to the output type.
* ``gemm_tile_ledger``: the per-K-iteration tile ledger of "GPU 执行模型",
  section "Tile 小账本".
* ``axpby`` / ``epilogue``: the epilogue variants C = act(alpha A.B + beta C
  + bias) in fp64, and ``fusion_saving_bytes``, the HBM bytes a fused
  epilogue saves ("GPU 执行模型", section "Fusion 的收益与上限").

Layouts: A is row-major M x K with leading dimension lda; B is stored K-major,
i.e. as an N x K array with leading dimension ldb (b(k,j) = B[j, k]); C is
row-major M x N.  Every function here is pinned by ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

from . import build as _build

_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        i64 = ctypes.c_int64
        vp = ctypes.c_void_p
        lib.oracle_gemm_f64.argtypes = [vp, i64, vp, i64, vp, i64, i64, i64, i64]
        lib.oracle_gemm_abs_f64.argtypes = [vp, i64, vp, i64, vp, i64, i64, i64, i64]
        lib.oracle_decode_bf16.argtypes = [vp, vp, i64]
        lib.oracle_decode_e4m3.argtypes = [vp, vp, i64]
        lib.oracle_decode_mx_operand.argtypes = [vp, i64, vp, i64, vp, i64, i64]
        lib.oracle_round_f32.argtypes = [vp, vp, i64]
        lib.oracle_round_bf16.argtypes = [vp, vp, i64]
        lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f64.restype = ctypes.c_double
        lib.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_f64.restype = ctypes.c_double
        lib.oracle_e8m0_to_f64.argtypes = [ctypes.c_uint8]
        lib.oracle_e8m0_to_f64.restype = ctypes.c_double
        lib.oracle_f64_to_bf16_rne.argtypes = [ctypes.c_double]
        lib.oracle_f64_to_bf16_rne.restype = ctypes.c_uint16
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        _LIB = lib
    return _LIB


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def num_threads() -> int:
    """OpenMP threads the oracle uses (all host cores unless limited)."""
    return int(_lib().oracle_num_threads())


def set_num_threads(n: int) -> None:
    _lib().oracle_set_num_threads(int(n))


# ------------------------------------------------------------------ codecs --

def decode_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16, any shape, C-contiguous) -> exact fp64."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, dtype=np.float64)
    _lib().oracle_decode_bf16(_ptr(bits), _ptr(out), bits.size)
    return out


def decode_e4m3(bits: np.ndarray) -> np.ndarray:
    """FP8 E4M3 codes (uint8) -> exact fp64."""
    bits = np.ascontiguousarray(bits, dtype=np.uint8)
    out = np.empty(bits.shape, dtype=np.float64)
    _lib().oracle_decode_e4m3(_ptr(bits), _ptr(out), bits.size)
    return out


def decode_e8m0(byte: int) -> float:
    return float(_lib().oracle_e8m0_to_f64(int(byte)))


def round_f32(c64: np.ndarray) -> np.ndarray:
    """fp64 -> binary32, round to nearest even."""
    c64 = np.ascontiguousarray(c64, dtype=np.float64)
    out = np.empty(c64.shape, dtype=np.float32)
    _lib().oracle_round_f32(_ptr(c64), _ptr(out), c64.size)
    return out


def round_bf16(c64: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 bit patterns (uint16), round to nearest even, directly."""
    c64 = np.ascontiguousarray(c64, dtype=np.float64)
    out = np.empty(c64.shape, dtype=np.uint16)
    _lib().oracle_round_bf16(_ptr(c64), _ptr(out), c64.size)
    return out


def f64_to_bf16_bits(x: float) -> int:
    return int(_lib().oracle_f64_to_bf16_rne(float(x)))


# -------------------------------------------------------------------- GEMM --

def _gemm_dense(a64: np.ndarray, b64: np.ndarray, absolute: bool) -> np.ndarray:
    a64 = np.ascontiguousarray(a64, dtype=np.float64)
    b64 = np.ascontiguousarray(b64, dtype=np.float64)
    M, K = a64.shape
    N, Kb = b64.shape
    if Kb != K:
        raise ValueError(f"A is {M}x{K} but B (stored N x K) is {N}x{Kb}")
    c = np.empty((M, N), dtype=np.float64)
    if M and N:
        fn = _lib().oracle_gemm_abs_f64 if absolute else _lib().oracle_gemm_f64
        fn(_ptr(a64), max(K, 1), _ptr(b64), max(K, 1), _ptr(c), N, M, N, K)
    return c


def gemm_f64(a64: np.ndarray, b64_nk: np.ndarray) -> np.ndarray:
    """C = A.B in fp64 for fp64 A (M x K) and B stored N x K."""
    return _gemm_dense(a64, b64_nk, absolute=False)


def gemm_abs_f64(a64: np.ndarray, b64_nk: np.ndarray) -> np.ndarray:
    """S[i][j] = sum_k |a(i,k) b(k,j)| (scales the parity tolerance)."""
    return _gemm_dense(a64, b64_nk, absolute=True)


def _bf16_operand(bits: np.ndarray, rows, K: int) -> np.ndarray:
    bits = np.asarray(bits, dtype=np.uint16)
    sub = bits[:, :K] if rows is None else bits[np.asarray(rows), :K]
    return decode_bf16(np.ascontiguousarray(sub))


def gemm_bf16_f64(a_bits: np.ndarray, b_bits: np.ndarray, K: int | None = None,
                  rows=None, cols=None, with_abs: bool = False):
    """Oracle GEMM over bf16 operands.

    a_bits: uint16 [M, lda] (row-major A, first K columns used);
    b_bits: uint16 [N, ldb] (K-major B, first K columns used).
    rows / cols: optional index arrays selecting a sub-block C[rows][:, cols]
    (used to check sampled outputs of full-size problems).
    Returns the fp64 sums (and the sum of |products| if with_abs).
    """
    if K is None:
        K = a_bits.shape[1]
    a64 = _bf16_operand(a_bits, rows, K)
    b64 = _bf16_operand(b_bits, cols, K)
    c = gemm_f64(a64, b64)
    if with_abs:
        return c, gemm_abs_f64(a64, b64)
    return c


def decode_mx_operand(codes: np.ndarray, scales: np.ndarray, K: int, rows=None) -> np.ndarray:
    """E4M3 codes [R, ldx] and E8M0 scales [R, >= K/32] -> fp64 values [R', K]."""
    if K % 32:
        raise ValueError("block-scaled operands need K to be a multiple of 32")
    codes = np.asarray(codes, dtype=np.uint8)
    scales = np.asarray(scales, dtype=np.uint8)
    if rows is not None:
        codes = codes[np.asarray(rows)]
        scales = scales[np.asarray(rows)]
    codes = np.ascontiguousarray(codes)
    scales = np.ascontiguousarray(scales)
    R = codes.shape[0]
    out = np.empty((R, K), dtype=np.float64)
    if R and K:
        _lib().oracle_decode_mx_operand(_ptr(codes), codes.shape[1], _ptr(scales),
                                        scales.shape[1], _ptr(out), R, K)
    return out


def gemm_mxfp8_f64(a_codes, sfa, b_codes, sfb, K: int | None = None,
                   rows=None, cols=None, with_abs: bool = False):
    """Oracle block-scaled GEMM.

    a_codes uint8 [M, lda] E4M3, sfa uint8 [M, K/32] E8M0,
    b_codes uint8 [N, ldb] E4M3 (K-major B), sfb uint8 [N, K/32] E8M0.
    C[i][j] = sum_k (e4m3(a_ik) 2^(sfa[i][k/32]-127)) (e4m3(b_jk) 2^(sfb[j][k/32]-127)).
    """
    if K is None:
        K = a_codes.shape[1]
    a64 = decode_mx_operand(a_codes, sfa, K, rows)
    b64 = decode_mx_operand(b_codes, sfb, K, cols)
    c = gemm_f64(a64, b64)
    if with_abs:
        return c, gemm_abs_f64(a64, b64)
    return c


# ------------------------------------------------------------- tile ledger --

@dataclass(frozen=True)
class TileLedger:
    """Bookkeeping for one K_t step of an M_t x N_t output tile.

    From "GPU 执行模型", section "Tile 小账本": the operand tiles of one
    reduction step hold M_t K_t + K_t N_t elements; read once from HBM they
    cost that many elements' bytes; the multi-stage SMEM ring holds `stages`
    copies; one multiply-add counts as 2 FLOPs.  Stages enlarge residency but
    never add HBM reads.  Accumulator, C traffic, padding and cache misses are
    left out, so the intensity is an optimistic bound.
    """
    smem_bytes: int
    flops: int
    hbm_bytes: int
    arithmetic_intensity: float
    fits_smem: bool


def gemm_tile_ledger(m_tile: int, n_tile: int, k_tile: int, element_bytes: int,
                     stages: int, smem_limit: int) -> TileLedger:
    dims = (m_tile, n_tile, k_tile, element_bytes, stages)
    if any(int(d) <= 0 for d in dims):
        raise ValueError(f"every tile dimension, the element size and the stage count must be positive: {dims}")
    per_step_elems = k_tile * (m_tile + n_tile)      # A tile M_t x K_t plus B tile K_t x N_t
    bytes_once = per_step_elems * element_bytes
    ring = bytes_once * stages
    work = 2 * m_tile * n_tile * k_tile
    return TileLedger(smem_bytes=ring, flops=work, hbm_bytes=bytes_once,
                      arithmetic_intensity=work / bytes_once,
                      fits_smem=ring <= smem_limit)


def smem_estimate_double_buffer(m_tile: int, n_tile: int, k_tile: int, stages: int) -> int:
    """The capacity estimate M_smem ~ 2 s (M_t K_t + K_t N_t) of "GPU 执行模型",
    section "Tile 的容量约束" -- read with 2 = bf16 bytes per element and
    s = the number of pipeline stages."""
    return 2 * stages * (m_tile * k_tile + k_tile * n_tile)


# ---------------------------------------------------- full-size properties --

def gemm_line_sums_f64(a64: np.ndarray, b64_nk: np.ndarray):
    """Row and column sums of C = A.B without forming C, for checking every
    output of a full-size product at once:

        sum_j C[i][j] = sum_k a(i,k) (sum_j b(k,j))     (row sums, length M)
        sum_i C[i][j] = sum_k (sum_i a(i,k)) b(k,j)     (column sums, length N)

    together with the matching magnitudes sum_j sum_k |a(i,k) b(k,j)| and
    sum_i sum_k |a(i,k) b(k,j)| that scale the per-element tolerance.
    All in fp64; each is a plain contraction (library matrix-vector products).
    """
    a64 = np.asarray(a64, dtype=np.float64)
    b64 = np.asarray(b64_nk, dtype=np.float64)
    b_col = b64.sum(axis=0)               # over j, for each k
    b_abs = np.abs(b64).sum(axis=0)
    a_row = a64.sum(axis=0)               # over i, for each k
    a_abs = np.abs(a64).sum(axis=0)
    rows = a64 @ b_col
    rows_mag = np.abs(a64) @ b_abs
    cols = b64 @ a_row
    cols_mag = np.abs(b64) @ a_abs
    return rows, rows_mag, cols, cols_mag


# ------------------------------------------------------- epilogue variants --

def axpby(c_ab64: np.ndarray, c_old64: np.ndarray, alpha: float, beta: float) -> np.ndarray:
    """C <- alpha (A.B) + beta C_old, in fp64, the BLAS-style reading of the
    epilogue variants (alpha/beta) of a GEMM: the old C is used only when
    beta != 0, so beta = 0 ignores whatever it holds (NaN included)."""
    c = float(alpha) * np.asarray(c_ab64, dtype=np.float64)
    if beta != 0.0:
        c = c + float(beta) * np.asarray(c_old64, dtype=np.float64)
    return c


ACT_NONE, ACT_RELU, ACT_GELU, ACT_GELU_TANH = 0, 1, 2, 3


def gelu(x: np.ndarray) -> np.ndarray:
    """x Phi(x), Phi the standard normal CDF, written with erf (fp64)."""
    from math import erf, sqrt
    x = np.asarray(x, dtype=np.float64)
    return x * 0.5 * (1.0 + np.vectorize(erf, otypes=[np.float64])(x / sqrt(2.0)))


def gelu_tanh(x: np.ndarray) -> np.ndarray:
    """The tanh form of GELU, 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))),
    in fp64 (Hendrycks and Gimpel, "Gaussian Error Linear Units", 2016)."""
    from math import pi, sqrt
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + np.tanh(sqrt(2.0 / pi) * (x + 0.044715 * x ** 3)))


def relu(x: np.ndarray) -> np.ndarray:
    """0 where x < 0, else x itself (NaN stays NaN)."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x < 0.0, 0.0, x)


def epilogue(c_ab64: np.ndarray, c_old64: np.ndarray, alpha: float, beta: float,
             bias64: np.ndarray | None, act: int) -> np.ndarray:
    """A fused GEMM epilogue, in fp64: act(alpha (A.B) + beta C_old + bias),
    the bias one value per column of C.  Its arithmetic is the pointwise
    sequence that fusion folds into the GEMM's write-back ("GPU 执行模型",
    section "Fusion 的收益与上限"); which pointwise ops to offer (bias, ReLU,
    GELU and its tanh form) is this library's choice."""
    c = axpby(c_ab64, c_old64, alpha, beta)
    if bias64 is not None:
        c = c + np.asarray(bias64, dtype=np.float64)[None, :]
    if act == ACT_RELU:
        return relu(c)
    if act == ACT_GELU:
        return gelu(c)
    if act == ACT_GELU_TANH:
        return gelu_tanh(c)
    if act != ACT_NONE:
        raise ValueError(f"unknown activation {act}")
    return c


def fusion_saving_bytes(intermediate_bytes: int) -> int:
    """HBM bytes saved by fusing a pointwise step into the producer: the
    intermediate tensor is neither written out nor read back, about
    2 M_intermediate ("GPU 执行模型", section "Fusion 的收益与上限")."""
    return 2 * int(intermediate_bytes)
