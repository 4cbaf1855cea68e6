"""GPU parity of the cluster split-K configurations: the S CTAs of a cluster
(S = 2, 4 or 8) compute one 128 x 128 or 128 x 256 tile together, each over
its own share of the K blocks, and member j sums column slice j of the tile
from every member's fp32 partial in member order, the partials crossing
through distributed shared memory.  Compared with the oracle element by
element; integer inputs bit-exact.

In this process S is chosen by shape (the shapes below reach 8, 4 and 2).  A
child process per S forces the factor (B200GEMM_KSPLIT, read once by the
library), which also reaches members whose share of K is empty (K of fewer
than S 64-wide blocks) and the fused epilogue and transposed operands on
every factor."""
import json
import os
import subprocess
import sys
import textwrap

import pytest

import oracle
from dense_gemm_engineering_bf16_b200 import gemm as G
from dense_gemm_engineering_bf16_b200 import synth

from gpu_helpers import assert_close, assert_exact, run_gemm

pytestmark = pytest.mark.gpu
F32, BF16 = G.OUT_F32, G.OUT_BF16
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SPLIT = ["1cta_128x128_splitk", "1cta_128x256_splitk"]


def _check(M, N, K, dist, workload, cfg, c_type=F32):
    ld = K + (-K % 8)                  # rows on 16-byte boundaries (TMA)
    a_bits, b_bits = synth.bf16_operands(M, N, K, dist, workload=workload, lda=ld, ldb=ld)
    C = run_gemm(a_bits, b_bits, M, N, K, c_type=c_type, config=cfg)
    got, guard_ok = C.download()
    assert guard_ok, "write outside C's M x N window"
    c_ref, s_abs = oracle.gemm_bf16_f64(a_bits, b_bits, K=K, with_abs=True)
    what = f"{cfg} {M}x{N}x{K}"
    if dist == "ints":
        assert_exact(got, c_ref, c_type, what)
    else:
        assert_close(got, c_ref, s_abs, c_type, what)
    return got


# (M, N, K): one tile with a long K (S = 8 for fp32 128 x 256), 32 and 64
# tiles (S = 4, 2), ragged M, N and K everywhere
SHAPES = [(100, 200, 4096), (1000, 1000, 1000), (1000, 2000, 777), (300, 300, 3000), (1, 129, 2048)]


@pytest.mark.parametrize("cfg", SPLIT)
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("c_type", [F32, BF16])
def test_integers_bit_exact(cfg, shape, c_type):
    M, N, K = shape
    _check(M, N, K, "ints", 500 + M % 97, cfg, c_type)


@pytest.mark.parametrize("cfg", SPLIT)
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("c_type", [F32, BF16])
def test_normal_within_tolerance(cfg, shape, c_type):
    M, N, K = shape
    _check(M, N, K, "normal", 520 + M % 89, cfg, c_type)


@pytest.mark.parametrize("cfg", SPLIT)
def test_deterministic(cfg):
    """The members' partials are added in member order whatever order they
    arrive in: repeated calls give the same bits."""
    M, N, K = 700, 900, 3000
    a_bits, b_bits = synth.bf16_operands(M, N, K, "normal", workload=540)
    first = run_gemm(a_bits, b_bits, M, N, K, config=cfg).bits()
    for _ in range(3):
        assert (run_gemm(a_bits, b_bits, M, N, K, config=cfg).bits() == first).all()


CHILD = textwrap.dedent(r"""
    import json, sys
    sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + "/tests")
    import numpy as np, torch
    import oracle
    from dense_gemm_engineering_bf16_b200 import gemm as G, synth
    from gpu_helpers import run_gemm, to_device_bf16, tolerance
    res = {}
    def record(name, ok, detail=""):
        res[name] = [bool(ok), detail]
    for cfg in ("1cta_128x128_splitk", "1cta_128x256_splitk"):
        for (M, N, K) in ((300, 260, 192), (200, 520, 64), (129, 257, 4096), (640, 384, 1000)):
            for ct in (G.OUT_F32, G.OUT_BF16):
                for dist in ("ints", "normal"):
                    a, b = synth.bf16_operands(M, N, K, dist, workload=560 + K % 31)
                    C = run_gemm(a, b, M, N, K, c_type=ct, config=cfg)
                    got, guard = C.download()
                    ref, s = oracle.gemm_bf16_f64(a, b, K=K, with_abs=True)
                    if dist == "ints":
                        want = oracle.round_f32(ref) if ct == G.OUT_F32 else oracle.decode_bf16(oracle.round_bf16(ref))
                        ok = guard and np.array_equal(got, np.asarray(want, dtype=np.float64))
                    else:
                        ok = guard and bool(np.all(np.abs(got - ref) <= tolerance(ref, s, ct)))
                    record(f"{cfg} {M}x{N}x{K} ct{ct} {dist}", ok)
        # fused epilogue (alpha, beta, bias, GELU) with B stored K x N
        M, N, K = 257, 264, 1536
        a, b = synth.bf16_operands(M, N, K, "normal", workload=580)
        bT = np.ascontiguousarray(b.T)
        c_old = synth.normal(581, (M, N))
        bias = synth.uniform(582, (N,)).astype(np.float32)
        C = torch.from_numpy(c_old.astype(np.float32)).cuda()
        G.gemm_force_config(cfg)
        try:
            G.gemm_bf16_fused(to_device_bf16(a), to_device_bf16(bT), C, M, N, K, K, N, N, G.OUT_F32, G.KMAJOR,
                              G.MNMAJOR, 0.5, -1.5, torch.from_numpy(bias).cuda(), G.ACT_GELU)
        finally:
            G.gemm_force_config("auto")
        G.gemm_check_device_status()
        got = C.cpu().numpy().astype(np.float64)
        ab, s = oracle.gemm_bf16_f64(a, b, with_abs=True)
        old = c_old.astype(np.float32).astype(np.float64)
        want = oracle.epilogue(ab, old, 0.5, -1.5, bias.astype(np.float64), G.ACT_GELU)
        lin = oracle.axpby(ab, old, 0.5, -1.5) + bias.astype(np.float64)[None, :]
        tol = 1.13 * (0.5 * (1e-3 * s + 1e-6) + 1e-6 * np.abs(1.5 * old)) + 1e-6 * np.abs(lin) + 1e-6
        record(f"{cfg} fused gelu B KxN", bool(np.all(np.abs(got - want) <= tol)))
    print(json.dumps(res))
""")


@pytest.mark.parametrize("ksplit", [2, 4, 8])
def test_forced_factor(ksplit):
    """Every split factor on both tiles, fp32 and bf16 C (where the slices
    stay whole store chunks; otherwise the shape's own choice runs), with K
    of 3 and 1 blocks (members with no share of K add zeros), ragged edges,
    and the fused epilogue with a transposed B."""
    env = dict(os.environ, B200GEMM_KSPLIT=str(ksplit))
    out = subprocess.run([sys.executable, "-c", CHILD, ROOT], env=env, capture_output=True, text=True,
                         timeout=600)
    assert out.returncode == 0, out.stdout[-2000:] + out.stderr[-4000:]
    res = json.loads(out.stdout.strip().splitlines()[-1])
    bad = {k: v for k, v in res.items() if not v[0]}
    assert not bad, bad
