"""The split tail of the square kernels (off by default; B200GEMM_SPLIT turns
it on): the last wave's tiles are cut into K parts whose fp32 partials the
last-arriving part sums in part order.  Run in child processes, since the
switch is read once per process; results must match the oracle, integers
bit-exactly, and repeat bit-identically."""
import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent(r"""
    import os, sys
    sys.path.insert(0, sys.argv[1]); sys.path.insert(0, os.path.join(sys.argv[1], "tests"))
    import numpy as np, torch
    import oracle
    from dense_gemm_engineering_bf16_b200 import gemm as G, synth
    from gpu_helpers import to_device_bf16
    cases = [("2cta_256x256_clc", 600, 520, 1000, "normal"), ("2cta_256x256", 4096, 2560, 512, "uniform"),
             ("1cta_128x128", 300, 200, 136, "ints"), ("1cta_128x256_clc", 257, 640, 2048, "normal")]
    for cfg, M, N, K, dist in cases:
        a, b = synth.bf16_operands(M, N, K, dist, workload=500 + M)
        A, B = to_device_bf16(a), to_device_bf16(b)
        G.gemm_force_config(cfg)
        outs = []
        for rep in range(2):
            C = torch.full((M, N + 4), float("nan"), dtype=torch.float32, device="cuda")
            G.gemm_bf16(A, B, C, M, N, K, K, K, N + 4, G.OUT_F32)
            G.gemm_check_device_status()
            outs.append(C.cpu().numpy().astype(np.float64))
        G.gemm_force_config("auto")
        assert np.array_equal(outs[0], outs[1], equal_nan=True), (cfg, "not repeatable")
        got = outs[0]
        assert np.isnan(got[:, N:]).all(), (cfg, "wrote past N")
        rows = np.arange(0, M, 37)
        ref, s = oracle.gemm_bf16_f64(a, b, rows=rows, with_abs=True)
        if dist == "ints":
            assert np.array_equal(got[rows, :N], oracle.round_f32(ref).astype(np.float64)), cfg
        else:
            assert np.all(np.abs(got[rows, :N] - ref) <= 1e-3 * s + 1e-6), cfg
        print(cfg, "ok", flush=True)
    print("split ok")
""")


@pytest.mark.parametrize("mode", ["auto", "3"])
def test_split_tail_matches_the_oracle(mode):
    env = dict(os.environ, B200GEMM_SPLIT=mode)
    out = subprocess.run([sys.executable, "-c", CHILD, ROOT], env=env, capture_output=True, text=True,
                         timeout=600)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "split ok" in out.stdout
