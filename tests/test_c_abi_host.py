"""The boundary from plain C: include/b200gemm.h compiles as C (not only
C++), a C program links against the library, and argument checks answer
through the C ABI before anything touches a device."""
import os
import shutil
import subprocess

import pytest

from dense_gemm_engineering_bf16_b200 import gemm as G

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_INC = "/usr/local/cuda/include"

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "b200gemm.h"

int main(void) {
    /* far-apart, 16-byte-aligned addresses that are never dereferenced:
       each call fails validation (or has nothing to do) first */
    void *A = (void *)0x7F0000000000ul, *B = (void *)0x7F0000100000ul, *C = (void *)0x7F0000200000ul;
    const uint8_t *sa = (const uint8_t *)0x7F0000300000ul, *sb = (const uint8_t *)0x7F0000400000ul;
    int s1 = gemm_bf16(A, B, C, -1, 8, 8, 8, 8, 8, GEMM_OUT_F32, 0);
    int s2 = gemm_bf16_ex(A, B, C, 8, 8, 8, 8, 8, 8, GEMM_OUT_F32, (gemm_layout_t)5, GEMM_LAYOUT_KMAJOR,
                          1.0f, 0.0f, 0);
    int s3 = gemm_bf16_fused(A, B, C, 8, 8, 8, 8, 8, 8, GEMM_OUT_BF16, GEMM_LAYOUT_KMAJOR, GEMM_LAYOUT_MNMAJOR,
                             1.0f, 0.0f, 0, (gemm_act_t)9, 0);
    int s4 = gemm_mxfp8(A, sa, B, sb, C, 8, 8, 48, 48, 48, 8, 0);   /* K not a multiple of 32 */
    int s5 = gemm_bf16(A, B, C, 0, 8, 8, 8, 8, 8, GEMM_OUT_F32, 0);
    printf("%d %d %d %d %d %d %s\n", s1, s2, s3, s4, s5, gemm_launches_per_call(4, 4, 32, 1),
           gemm_status_string(GEMM_ERR_MISALIGNED));
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None or not os.path.isdir(CUDA_INC), reason="needs gcc and CUDA headers")
def test_header_compiles_as_c_and_links(tmp_path):
    src = tmp_path / "abi.c"
    exe = tmp_path / "abi"
    src.write_text(PROGRAM)
    libdir = os.path.dirname(G.library_path)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-I", CUDA_INC,
                    str(src), "-L", libdir, "-lb200gemm", "-o", str(exe)], check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True,
                         env=dict(os.environ, LD_LIBRARY_PATH=libdir)).stdout.split(" ", 6)
    assert out[:6] == ["1", "1", "1", "1", "0", "2"]      # invalid x4, empty problem OK, 2 launches (MXFP8)
    assert out[6].startswith("GEMM_ERR_MISALIGNED")
