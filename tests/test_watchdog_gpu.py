"""Failure detection without a GPU fault: every mbarrier wait in the kernels
is bounded.  A test-only switch makes CTA 0 leave one pipeline stage unarmed
(a barrier nothing will complete); the MMA warp's wait expires after the
watchdog limit, every role of the CTA (and of its pair) leaves its loop, the
kernel frees TMEM and exits, and gemm_check_device_status() reports
GEMM_ERR_TIMEOUT with the role and CTA.  The context stays usable: the next
call on the same stream is correct.

The switch, B200GEMM_INJECT_TIMEOUT, is a per-launch mask ('1' = inject into
that launch) that the library reads once; the short watchdog limit is read
once too.  Both are set in a child process's environment, so they apply only
there.  The child alternates an injected and a clean launch per
configuration, then does the same through gemm_bf16_noalloc, whose status
block is the library's static scratch array."""
import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CFGS = ("1cta_128x128", "2cta_256x256", "2cta_256x256_clc", "2cta_512x256_clc", "1cta_128x256_splitk")

CHILD = textwrap.dedent(r"""
    import os, sys, time
    sys.path.insert(0, sys.argv[1]); sys.path.insert(0, os.path.join(sys.argv[1], "tests"))
    import numpy as np, torch
    import oracle
    from dense_gemm_engineering_bf16_b200 import gemm as G, synth
    from gpu_helpers import to_device_bf16
    M = N = K = 768                   # past the latency path (which has no waits to bound)
    a, b = synth.bf16_operands(M, N, K, "normal", workload=77)
    A, B = to_device_bf16(a), to_device_bf16(b)
    C = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    ref, s = oracle.gemm_bf16_f64(a, b, with_abs=True)
    entries = [(cfg, G.gemm_bf16) for cfg in sys.argv[2].split(",")] + [("auto", G.gemm_bf16_noalloc)]
    for cfg, fn in entries:
        name = fn.__name__ + ":" + cfg
        G.gemm_force_config(cfg)
        t0 = time.time()
        fn(A, B, C, M, N, K, K, K, N, G.OUT_F32)          # injected launch
        st = G.gemm_check_device_status(check=False)
        dt = time.time() - t0
        where, block = G.gemm_last_timeout_detail()
        assert st == 6, (name, st)
        assert where == 2 * 16 + 1 and block == 0, (name, where, block)   # MMA warp, full barrier, CTA 0
        assert dt < 5.0, dt
        assert G.gemm_check_device_status(check=False) == 0, name        # reading cleared it
        C.zero_()
        fn(A, B, C, M, N, K, K, K, N, G.OUT_F32)          # clean launch
        assert G.gemm_check_device_status(check=False) == 0, name
        got = C.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got - ref) <= 1e-3 * s + 1e-6), name
        print(name, "timeout reported in %.3f s, next call correct" % dt, flush=True)
    print("watchdog ok")
""")


def test_dropped_arrival_times_out_cleanly_and_context_survives():
    launches = len(CFGS) + 1                  # each configuration, then gemm_bf16_noalloc
    env = dict(os.environ, B200GEMM_WATCHDOG_MS="100", B200GEMM_INJECT_TIMEOUT="10" * launches)
    out = subprocess.run([sys.executable, "-c", CHILD, ROOT, ",".join(CFGS)], env=env, capture_output=True,
                         text=True, timeout=300)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "watchdog ok" in out.stdout
