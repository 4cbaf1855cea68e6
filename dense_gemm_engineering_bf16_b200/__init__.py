"""B200-native dense GEMM: C = A.B with bf16 inputs / fp32 accumulation, and a
block-scaled MXFP8 variant, as hand-written sm_100a kernels behind a C ABI.

The binding (``gemm_bf16``, ``gemm_mxfp8``, ``gemm_check_device_status``,
``gemm_status_string`` ...) is loaded on first attribute access, so that
``synth`` can be imported on machines without the built library.  Accessing
a binding name when the library is missing raises immediately: there is no
fallback path.
"""
from importlib import import_module

_BINDING_NAMES = {
    "gemm_bf16", "gemm_bf16_ex", "gemm_bf16_fused", "gemm_bf16_noalloc", "gemm_mxfp8", "gemm_check_device_status", "gemm_status_string",
    "gemm_force_config", "gemm_select_config", "gemm_launches_per_call",
    "gemm_last_timeout_detail", "GemmError", "OUT_F32", "OUT_BF16", "KMAJOR", "MNMAJOR", "ACT_NONE", "ACT_RELU",
    "ACT_GELU", "ACT_GELU_TANH", "CONFIGS",
    "STATUS_NAMES", "lib", "library_path",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        return getattr(import_module(".gemm", __name__), name)
    raise AttributeError(name)
