"""ctypes binding of the C ABI in ``include/b200gemm.h``.

Argument marshalling only: tensors become device pointers, streams become
``cudaStream_t`` handles, and a non-OK status becomes ``GemmError``.  Every
step of the computation runs in the library's kernels.  Importing this module
without the built library raises -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(PKG, "libb200gemm.so")

if not os.path.exists(library_path):
    raise ImportError(
        f"{library_path} is missing: build it with "
        "`python -m dense_gemm_engineering_bf16_b200.build` (nvcc, sm_100a)")

lib = ctypes.CDLL(library_path)

OUT_F32 = 0
OUT_BF16 = 1
KMAJOR = 0      # A as M x K, B as N x K
MNMAJOR = 1     # A as K x M, B as K x N (row-major K x N)
ACT_NONE = 0
ACT_RELU = 1
ACT_GELU = 2
ACT_GELU_TANH = 3

CONFIGS = {
    "auto": 0,
    "1cta_128x256": 1,
    "1cta_128x128": 2,
    "2cta_256x256": 3,
    "skinny": 4,
    "2cta_256x256_clc": 5,
    "1cta_128x256_clc": 6,
    "mxfp8_1cta_128x256": 7,
    "mxfp8_2cta_256x256": 8,
    "2cta_512x256_clc": 9,
    "2cta_256x256_sk": 10,
    "2cta_256x224": 11,
    "1cta_128x128_splitk": 12,
    "1cta_128x256_splitk": 13,
    "small": 14,
}

STATUS_NAMES = {
    0: "GEMM_OK", 1: "GEMM_ERR_INVALID_VALUE", 2: "GEMM_ERR_MISALIGNED", 3: "GEMM_ERR_ALIAS",
    4: "GEMM_ERR_UNSUPPORTED_DEVICE", 5: "GEMM_ERR_LAUNCH", 6: "GEMM_ERR_TIMEOUT",
    7: "GEMM_ERR_TOO_LARGE", 8: "GEMM_ERR_CAPTURE",
}

_i64 = ctypes.c_int64
_vp = ctypes.c_void_p
_int = ctypes.c_int

lib.gemm_bf16.argtypes = [_vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i64, _int, _vp]
lib.gemm_bf16.restype = _int
lib.gemm_bf16_noalloc.argtypes = [_vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i64, _int, _vp]
lib.gemm_bf16_noalloc.restype = _int
lib.gemm_bf16_ex.argtypes = [_vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i64, _int, _int, _int,
                             ctypes.c_float, ctypes.c_float, _vp]
lib.gemm_bf16_ex.restype = _int
lib.gemm_bf16_fused.argtypes = [_vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i64, _int, _int, _int,
                                ctypes.c_float, ctypes.c_float, _vp, _int, _vp]
lib.gemm_bf16_fused.restype = _int
lib.gemm_bf16_allgather.argtypes = [_vp, _vp, ctypes.POINTER(_vp), _int, _i64, _i64, _i64, _i64, _i64, _i64,
                                    _i64, _int, _vp]
lib.gemm_bf16_allgather.restype = _int
lib.gemm_mxfp8.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i64, _vp]
lib.gemm_mxfp8.restype = _int
lib.gemm_check_device_status.argtypes = [_vp]
lib.gemm_check_device_status.restype = _int
lib.gemm_last_timeout_detail.argtypes = [ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)]
lib.gemm_last_timeout_detail.restype = None
lib.gemm_status_string.argtypes = [_int]
lib.gemm_status_string.restype = ctypes.c_char_p
lib.gemm_last_cuda_error.argtypes = []
lib.gemm_last_cuda_error.restype = _int
lib.gemm_force_config.argtypes = [_int]
lib.gemm_force_config.restype = _int
lib.gemm_select_config.argtypes = [_i64, _i64, _i64]
lib.gemm_select_config.restype = _int
lib.gemm_launches_per_call.argtypes = [_i64, _i64, _i64, _int]
lib.gemm_launches_per_call.restype = _int


class GemmError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = int(status)
        msg = gemm_status_string(self.status)
        if self.status == 5:
            msg += f" (CUDA error {lib.gemm_last_cuda_error()})"
        super().__init__(f"{where}: {msg}" if where else msg)


def gemm_status_string(status: int) -> str:
    return lib.gemm_status_string(int(status)).decode()


def _ptr(x) -> int:
    if x is None:
        return 0
    if isinstance(x, int):
        return x
    return int(x.data_ptr())


def _stream(s) -> int:
    if s is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(s, int):
        return s
    return int(s.cuda_stream)


def _check(status: int, where: str, check: bool) -> int:
    if check and status != 0:
        raise GemmError(status, where)
    return status


def gemm_bf16(A, B, C, M: int, N: int, K: int, lda: int, ldb: int, ldc: int,
              c_type: int = OUT_F32, stream=None, check: bool = True) -> int:
    """C = A.B (bf16 A row-major M x K, bf16 B stored N x K, C M x N of c_type).

    A, B, C: torch tensors (device) or raw device pointers; stream: a
    torch.cuda.Stream, a raw handle, or None for torch's current stream.
    """
    st = lib.gemm_bf16(_ptr(A), _ptr(B), _ptr(C), M, N, K, lda, ldb, ldc, int(c_type), _stream(stream))
    return _check(st, "gemm_bf16", check)


def gemm_bf16_ex(A, B, C, M: int, N: int, K: int, lda: int, ldb: int, ldc: int,
                 c_type: int = OUT_F32, a_layout: int = KMAJOR, b_layout: int = KMAJOR,
                 alpha: float = 1.0, beta: float = 0.0, stream=None, check: bool = True) -> int:
    """C = alpha * A.B + beta * C with K-major or MN-major operands
    (see include/b200gemm.h, gemm_bf16_ex)."""
    st = lib.gemm_bf16_ex(_ptr(A), _ptr(B), _ptr(C), M, N, K, lda, ldb, ldc, int(c_type), int(a_layout),
                          int(b_layout), float(alpha), float(beta), _stream(stream))
    return _check(st, "gemm_bf16_ex", check)


def gemm_bf16_fused(A, B, C, M: int, N: int, K: int, lda: int, ldb: int, ldc: int,
                    c_type: int = OUT_F32, a_layout: int = KMAJOR, b_layout: int = KMAJOR,
                    alpha: float = 1.0, beta: float = 0.0, bias=None, act: int = ACT_NONE,
                    stream=None, check: bool = True) -> int:
    """C = act(alpha * A.B + beta * C + bias) with bias one fp32 value per
    column of C, fused into the GEMM's write-back (see include/b200gemm.h,
    gemm_bf16_fused)."""
    st = lib.gemm_bf16_fused(_ptr(A), _ptr(B), _ptr(C), M, N, K, lda, ldb, ldc, int(c_type), int(a_layout),
                             int(b_layout), float(alpha), float(beta), _ptr(bias) if bias is not None else None,
                             int(act), _stream(stream))
    return _check(st, "gemm_bf16_fused", check)


def gemm_bf16_allgather(A, B, C_dst, M: int, N: int, K: int, lda: int, ldb: int, ldc: int, row0: int,
                        c_type: int = OUT_F32, stream=None, check: bool = True) -> int:
    """This GPU's slab C[row0:row0+M] = A.B written into every C of C_dst
    (this GPU's own C first, then other GPUs' mapped C buffers): a row-
    sharded GEMM with its all-gather in the write-back (see
    include/b200gemm.h, gemm_bf16_allgather)."""
    ptrs = (_vp * len(C_dst))(*[_ptr(c) for c in C_dst])
    st = lib.gemm_bf16_allgather(_ptr(A), _ptr(B), ptrs, len(C_dst), M, N, K, lda, ldb, ldc, row0, int(c_type),
                                 _stream(stream))
    return _check(st, "gemm_bf16_allgather", check)


def gemm_mxfp8(A, sfa, B, sfb, C, M: int, N: int, K: int, lda: int, ldb: int, ldc: int,
               stream=None, check: bool = True) -> int:
    """Block-scaled C = (sa.A).(sb.B): E4M3 A (M x lda bytes), E4M3 B stored
    N x ldb, E8M0 scales sfa (M x K/32) and sfb (N x K/32), bf16 C (M x ldc)."""
    st = lib.gemm_mxfp8(_ptr(A), _ptr(sfa), _ptr(B), _ptr(sfb), _ptr(C), M, N, K, lda, ldb, ldc,
                        _stream(stream))
    return _check(st, "gemm_mxfp8", check)


def gemm_bf16_noalloc(A, B, C, M: int, N: int, K: int, lda: int, ldb: int, ldc: int,
                      c_type: int = OUT_F32, stream=None, check: bool = True) -> int:
    """gemm_bf16 without any device allocation: the kernels' scratch is a
    static array inside the library (see include/b200gemm.h)."""
    st = lib.gemm_bf16_noalloc(_ptr(A), _ptr(B), _ptr(C), M, N, K, lda, ldb, ldc, int(c_type),
                               _stream(stream))
    return _check(st, "gemm_bf16_noalloc", check)


def gemm_check_device_status(stream=None, check: bool = True) -> int:
    st = lib.gemm_check_device_status(_stream(stream))
    return _check(st, "gemm_check_device_status", check)


def gemm_last_timeout_detail():
    w = ctypes.c_int32()
    b = ctypes.c_int32()
    lib.gemm_last_timeout_detail(ctypes.byref(w), ctypes.byref(b))
    return int(w.value), int(b.value)


def gemm_force_config(config) -> None:
    cid = CONFIGS[config] if isinstance(config, str) else int(config)
    _check(lib.gemm_force_config(cid), "gemm_force_config", True)


def gemm_select_config(M: int, N: int, K: int) -> int:
    return int(lib.gemm_select_config(M, N, K))


def gemm_launches_per_call(M: int, N: int, K: int, block_scaled: bool = False) -> int:
    return int(lib.gemm_launches_per_call(M, N, K, int(bool(block_scaled))))
