"""Failure detection without a GPU fault: every mbarrier wait in the kernels
is bounded.  A test-only switch makes CTA 0 leave one pipeline stage unarmed
(a barrier nothing will complete); the MMA warp's wait expires after the
watchdog limit, every role of the CTA (and of its pair) leaves its loop, the
kernel frees TMEM and exits, and gemm_check_device_status() reports
GEMM_ERR_TIMEOUT with the role and CTA.  The context stays usable: the next
call on the same stream is correct.

Runs in a child process so that the short watchdog limit (read once when the
library starts) applies only there."""
import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent(r"""
    import os, sys, time
    sys.path.insert(0, sys.argv[1]); sys.path.insert(0, os.path.join(sys.argv[1], "tests"))
    import numpy as np, torch
    import oracle
    from dense_gemm_engineering_bf16_b200 import gemm as G, synth
    from gpu_helpers import to_device_bf16
    M = N = K = 512
    a, b = synth.bf16_operands(M, N, K, "normal", workload=77)
    A, B = to_device_bf16(a), to_device_bf16(b)
    C = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    ref, s = oracle.gemm_bf16_f64(a, b, with_abs=True)
    for cfg in ("1cta_128x128", "2cta_256x256", "2cta_256x256_clc", "2cta_512x256_clc"):
        G.gemm_force_config(cfg)
        os.environ["B200GEMM_INJECT_TIMEOUT"] = "1"
        t0 = time.time()
        G.gemm_bf16(A, B, C, M, N, K, K, K, N, G.OUT_F32)
        st = G.gemm_check_device_status(check=False)
        dt = time.time() - t0
        where, block = G.gemm_last_timeout_detail()
        assert st == 6, (cfg, st)
        assert where == 2 * 16 + 1 and block == 0, (cfg, where, block)   # MMA warp, full barrier, CTA 0
        assert dt < 5.0, dt
        os.environ["B200GEMM_INJECT_TIMEOUT"] = "0"
        C.zero_()
        G.gemm_bf16(A, B, C, M, N, K, K, K, N, G.OUT_F32)
        assert G.gemm_check_device_status(check=False) == 0
        got = C.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got - ref) <= 1e-3 * s + 1e-6), cfg
        print(cfg, "timeout reported in %.3f s, next call correct" % dt, flush=True)
    print("watchdog ok")
""")


def test_dropped_arrival_times_out_cleanly_and_context_survives():
    env = dict(os.environ, B200GEMM_WATCHDOG_MS="100")
    out = subprocess.run([sys.executable, "-c", CHILD, ROOT], env=env, capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "watchdog ok" in out.stdout
