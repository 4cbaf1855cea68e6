"""The C-ABI boundary on the host: the library loads, exports every symbol
the public header declares, and rejects bad arguments with the documented
status before anything is queued.  No kernel is launched here (CPU only)."""
import ctypes
import glob
import os
import re
import subprocess

import pytest
import torch

from dense_gemm_engineering_bf16_b200 import gemm as G

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))


def _declared():
    names = []
    for h in HEADERS:
        text = open(h).read()
        names += re.findall(r"^B200GEMM_API\s+[\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M)
    return names


def test_header_declares_and_library_exports_everything():
    names = _declared()
    assert "gemm_bf16" in names and "gemm_check_device_status" in names
    out = subprocess.run(["nm", "-D", "--defined-only", G.library_path], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(\w+)$", out, flags=re.M))
    missing = [n for n in names if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    for n in names:
        assert hasattr(G.lib, n)


A = 0x7F0000000000   # never dereferenced: every call below fails validation first
B = 0x7F0000100000
C = 0x7F0000200000


def _call(A_=A, B_=B, C_=C, M=128, N=128, K=128, lda=None, ldb=None, ldc=None, ct=G.OUT_F32):
    lda = K if lda is None else lda
    ldb = K if ldb is None else ldb
    ldc = N if ldc is None else ldc
    return G.lib.gemm_bf16(A_, B_, C_, M, N, K, lda, ldb, ldc, ct, 0)


def test_rejects_bad_arguments_before_any_launch():
    assert _call(M=-1) == 1
    assert _call(K=-5) == 1
    assert _call(ct=7) == 1
    assert _call(lda=64) == 1                       # lda < K
    assert _call(ldb=100) == 1                      # ldb < K
    assert _call(ldc=64) == 1                       # ldc < N
    assert _call(C_=0) == 1                         # null C
    assert _call(A_=0) == 1                         # null A with K > 0
    assert _call(A_=A + 2) == 2                     # misaligned pointer
    assert _call(C_=C + 8) == 2
    assert _call(K=100, lda=100, ldb=104) == 2      # 200-byte row pitch
    assert _call(N=100, ldc=102) == 2               # 408-byte fp32 pitch
    assert _call(N=100, ldc=100, ct=G.OUT_BF16) == 2   # 200-byte bf16 pitch
    assert _call(M=1 << 31) == 7
    assert _call(C_=A + 4096) == 3                  # C overlaps A
    assert _call(C_=B) == 3                         # C overlaps B


def _call_ex(A_=A, B_=B, C_=C, M=128, N=96, K=64, lda=None, ldb=None, ldc=None, ct=G.OUT_F32,
             al=G.KMAJOR, bl=G.KMAJOR, alpha=1.0, beta=0.0):
    lda = (M if al == G.MNMAJOR else K) if lda is None else lda
    ldb = (N if bl == G.MNMAJOR else K) if ldb is None else ldb
    ldc = N if ldc is None else ldc
    return G.lib.gemm_bf16_ex(A_, B_, C_, M, N, K, lda, ldb, ldc, ct, al, bl, alpha, beta, 0)


def test_ex_rejects_bad_layouts_and_pitches_before_any_launch():
    assert _call_ex(al=2) == 1 and _call_ex(bl=-1) == 1 and _call_ex(ct=3) == 1
    # A stored K x M: the pitch covers M, not K
    assert _call_ex(al=G.MNMAJOR, lda=64) == 1              # lda < M = 128
    assert _call_ex(al=G.MNMAJOR, M=100, lda=100) == 2       # 200-byte pitch
    assert _call_ex(bl=G.MNMAJOR, ldb=64) == 1               # ldb < N = 96
    assert _call_ex(bl=G.MNMAJOR, N=90, ldb=90, ldc=92) == 2  # 180-byte pitch
    # a K x M A of 64 rows with pitch 128 spans 16 KiB; C placed inside it aliases
    assert _call_ex(al=G.MNMAJOR, C_=A + 8192) == 3
    # K = 0 reads no operand: null A and B are fine, and C alone is validated
    assert _call_ex(K=0, A_=0, B_=0, C_=0) == 1
    assert _call_ex(K=0, A_=0, B_=0, C_=C + 4) == 2


def test_fused_rejects_bad_bias_and_activation_before_any_launch():
    f = G.lib.gemm_bf16_fused
    bias = 0x7F0000500000

    def call(bias_=bias, act=G.ACT_GELU, C_=C, K=64):
        return f(A, B, C_, 128, 96, K, 64, 64, 96, G.OUT_F32, G.KMAJOR, G.KMAJOR, 1.0, 0.0, bias_, act, 0)
    assert call(act=4) == 1 and call(act=-1) == 1
    assert call(bias_=bias + 4) == 2                 # bias not 16-byte aligned
    assert call(bias_=C + 128 * 4) == 3              # bias inside C's first rows
    assert call(K=0, bias_=bias + 8) == 2            # checked for K = 0 as well
    assert f(A, B, C, 0, 96, 64, 64, 64, 96, 0, 0, 0, 1.0, 0.0, bias + 4, 1, 0) == 0   # empty: nothing checked


def test_mxfp8_rejects_bad_arguments_before_any_launch():
    f = G.lib.gemm_mxfp8
    sa, sb = 0x7F0000300000, 0x7F0000400000
    assert f(A, sa, B, sb, C, 64, 64, 48, 48, 48, 64, 0) == 1          # K % 32
    assert f(A, sa, B, sb, C, 64, 64, 64, 40, 64, 64, 0) == 1          # lda < K
    assert f(A, sa, B, sb, C, 64, 64, 96, 104, 96, 64, 0) == 2         # lda not 16-byte multiple
    assert f(A, 0, B, sb, C, 64, 64, 64, 64, 64, 64, 0) == 1           # null scales
    assert f(A, sa, B, sb, sa, 64, 64, 64, 64, 64, 64, 0) == 3         # C overlaps sfa
    assert f(A, sa, B, sb, C, 0, 64, 64, 64, 64, 64, 0) == 0           # empty


def test_empty_problems_succeed_without_touching_memory():
    assert _call(M=0) == 0
    assert _call(N=0) == 0
    assert _call(M=0, A_=0, B_=0, C_=0) == 0
    assert G.gemm_launches_per_call(0, 5, 5) == 0
    assert G.gemm_launches_per_call(5, 5, 0) == 1
    assert G.gemm_launches_per_call(5, 5, 64, block_scaled=True) == 2
    assert G.gemm_launches_per_call(5, 5, 0, block_scaled=True) == 1


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_a_device_reports_unsupported_device():
    assert _call() == 4
    assert G.gemm_check_device_status(stream=0, check=False) in (0, 5)


def test_status_strings_and_config_control():
    for code, name in G.STATUS_NAMES.items():
        assert G.gemm_status_string(code).startswith(name)
    assert "unknown" in G.gemm_status_string(99)
    assert G.lib.gemm_force_config(99) == 1
    G.gemm_force_config("2cta_256x256")
    assert G.gemm_select_config(16, 16, 16) == G.CONFIGS["2cta_256x256"]
    G.gemm_force_config("2cta_512x256_clc")
    assert G.gemm_select_config(16, 16, 16) == G.CONFIGS["2cta_512x256_clc"]
    G.gemm_force_config("mxfp8_2cta_256x256")          # a block-scaled choice leaves bf16 on auto
    assert G.gemm_select_config(8192, 8192, 8192) == G.CONFIGS["2cta_512x256_clc"]
    G.gemm_force_config("auto")
    # long K, >= a wave of 512 x 256 tiles: the two-consumer tile
    assert G.gemm_select_config(8192, 8192, 8192) == G.CONFIGS["2cta_512x256_clc"]
    assert G.gemm_select_config(6144, 6144, 8192) == G.CONFIGS["2cta_512x256_clc"]
    assert G.gemm_select_config(1000, 8192, 8192) == G.CONFIGS["2cta_512x256_clc"]   # 64 tiles, 0.86 wave
    # K < 8192: its unhidden drain costs more than the shared B saves
    assert G.gemm_select_config(4096, 4096, 4096) == G.CONFIGS["2cta_256x256_clc"]
    assert G.gemm_select_config(1536, 8192, 8192) == G.CONFIGS["2cta_256x256_clc"]   # 96 tall tiles: 2 waves
    # K <= 2048: the static pair schedule
    assert G.gemm_select_config(4000, 3000, 2000) == G.CONFIGS["2cta_256x256"]
    assert G.gemm_select_config(2048, 8192, 2048) == G.CONFIGS["2cta_256x256"]
    assert G.gemm_select_config(8192, 8192, 1024) == G.CONFIGS["2cta_256x256"]
    # up to two waves of one-CTA 128 x 256 tiles: their lower fixed cost wins
    assert G.gemm_select_config(2048, 2048, 2048) == G.CONFIGS["1cta_128x256"]
    assert G.gemm_select_config(2560, 3584, 2048) == G.CONFIGS["1cta_128x256"]
    # a tiny product (at most 2^27 multiply-adds, K <= 2048, C of at most 2^20
    # elements): the latency path
    assert G.gemm_select_config(128, 128, 128) == G.CONFIGS["small"]
    assert G.gemm_select_config(300, 1000, 64) == G.CONFIGS["small"]
    assert G.gemm_select_config(512, 512, 512) == G.CONFIGS["small"]
    assert G.gemm_select_config(128, 128, 2048) == G.CONFIGS["small"]
    assert G.gemm_select_config(128, 256, 4096) == G.CONFIGS["1cta_128x128_splitk"]   # K > 2048
    assert G.gemm_select_config(2048, 2048, 32) != G.CONFIGS["small"]                   # C too wide
    # every 128 x 128 tile on an SM of its own
    assert G.gemm_select_config(1000, 1000, 1000) == G.CONFIGS["1cta_128x128"]   # K < 2048: no split
    assert G.gemm_select_config(1024, 1024, 256) == G.CONFIGS["1cta_128x128"]    # 2^28: past the latency path
    # tiles for at most half the SMs and K >= 2048: cluster split-K
    assert G.gemm_select_config(64, 4096, 4096) == G.CONFIGS["1cta_128x128_splitk"]
    assert G.gemm_select_config(48, 8192, 4096) == G.CONFIGS["1cta_128x128_splitk"]
    assert G.gemm_select_config(64, 8192, 8192) == G.CONFIGS["1cta_128x128_splitk"]
    assert G.gemm_select_config(256, 4096, 4096) == G.CONFIGS["1cta_128x128_splitk"]    # 64 tiles
    assert G.gemm_select_config(256, 8192, 8192) == G.CONFIGS["1cta_128x256_splitk"]    # 128; 64 wide
    assert G.gemm_select_config(512, 4096, 4096) == G.CONFIGS["1cta_128x256_splitk"]
    # a few rows and a long K: the skinny (swapped A/B) kernel
    assert G.gemm_select_config(16, 8192, 8192) == G.CONFIGS["skinny"]
    assert G.gemm_select_config(32, 2048, 8192) == G.CONFIGS["skinny"]
    assert G.gemm_select_config(32, 4096, 4096) == G.CONFIGS["skinny"]
    assert G.gemm_select_config(32, 4096, 2048) == G.CONFIGS["1cta_128x128_splitk"]
    # the 256 x 224 and stream-K configurations are never chosen by shape
    seen = {G.gemm_select_config(m, n, k) for m in (1, 100, 300, 1000, 3000, 8192)
            for n in (64, 1000, 3000, 8192) for k in (16, 1000, 5000, 16384)}
    assert G.CONFIGS["2cta_256x224"] not in seen and G.CONFIGS["2cta_256x256_sk"] not in seen
    with pytest.raises(G.GemmError):
        G.gemm_bf16(A, B, C, -1, 1, 1, 1, 1, 1, stream=0)


def test_binding_constants_match_the_header():
    text = "".join(open(h).read() for h in HEADERS)
    enum = {name.upper(): int(v) for name, v in re.findall(r"\b(GEMM_[A-Z0-9_x]+)\s*=\s*(\d+)", text)}
    for name, v in G.CONFIGS.items():
        assert enum["GEMM_CFG_" + name.upper()] == v, name
    assert enum["GEMM_CFG_COUNT_"] == max(G.CONFIGS.values()) + 1
    for name in ("NONE", "RELU", "GELU", "GELU_TANH"):
        assert enum["GEMM_ACT_" + name] == getattr(G, "ACT_" + name)
    assert (enum["GEMM_LAYOUT_KMAJOR"], enum["GEMM_LAYOUT_MNMAJOR"]) == (G.KMAJOR, G.MNMAJOR)
    assert (enum["GEMM_OUT_F32"], enum["GEMM_OUT_BF16"]) == (G.OUT_F32, G.OUT_BF16)
    for code, name in G.STATUS_NAMES.items():
        assert enum[name] == code


def test_configuration_choice_respects_its_own_rules():
    """Over a grid of shapes, the shape-based choice keeps to the rules its
    cost model was fitted under: the skinny kernel only for M <= 32 with a
    long K, split-K only with K >= 2048 and tiles for at most half the SMs,
    the single-buffered 512 x 256 tile only for K >= 8192, one-CTA 128 x 256
    tiles for at most two waves, the latency path exactly for the products of
    at most 2^27 multiply-adds with K <= 2048 and C of at most 2^20 elements,
    and never the forced-only kernels."""
    G.gemm_force_config("auto")
    C = G.CONFIGS
    cdiv = lambda a, b: -(-a // b)  # noqa: E731
    for M in (1, 16, 32, 33, 64, 100, 256, 300, 512, 1000, 2048, 4096, 8192):
        for N in (64, 256, 1000, 2048, 4096, 8192, 16384):
            for K in (16, 512, 1024, 2048, 4096, 8192, 16384):
                c = G.gemm_select_config(M, N, K)
                assert c in C.values() and c not in (C["auto"], C["2cta_256x224"], C["2cta_256x256_sk"]), (M, N, K)
                if c == C["skinny"]:
                    assert M <= 32 and K >= 4096, (M, N, K)
                if c in (C["1cta_128x128_splitk"], C["1cta_128x256_splitk"]):
                    assert K >= 2048, (M, N, K)
                    width = 128 if c == C["1cta_128x128_splitk"] else 256
                    assert cdiv(M, 128) * cdiv(N, width) <= 74, (M, N, K)
                if c in (C["2cta_512x256_clc"], C["1cta_128x256_clc"]):
                    assert K >= 8192, (M, N, K)
                if c == C["1cta_128x256"]:
                    assert cdiv(M, 128) * cdiv(N, 256) <= 2 * 148, (M, N, K)
                assert (c == C["small"]) == (M * N * K <= 1 << 27 and K <= 2048 and M * N <= 1 << 20), (M, N, K)
