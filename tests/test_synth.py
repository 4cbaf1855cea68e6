"""The seeded input generators: deterministic, the published splitmix64
stream, and the value ranges each workload recipe asks for.  CPU only."""
import numpy as np

import oracle
from dense_gemm_engineering_bf16_b200 import synth


def test_splitmix64_published_stream():
    # splitmix64 started at state 0: the first outputs of the reference generator
    got = synth.splitmix64(0, 3)
    assert [int(x) for x in got] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
    # offsets continue the same stream
    assert np.array_equal(synth.splitmix64(0, 2, offset=1), got[1:])


def test_deterministic_and_distinct_seeds():
    a1, b1 = synth.bf16_operands(33, 17, 40, "normal", workload=2)
    a2, b2 = synth.bf16_operands(33, 17, 40, "normal", workload=2)
    a3, _ = synth.bf16_operands(33, 17, 40, "normal", workload=3)
    assert np.array_equal(a1, a2) and np.array_equal(b1, b2)
    assert not np.array_equal(a1, a3)
    assert not np.array_equal(a1[:17], b1[:, :40][:17])


def test_value_ranges():
    u = oracle.decode_bf16(synth.bf16_operands(64, 64, 256, "uniform", workload=1)[0])
    assert u.min() >= -1 and u.max() <= 1 and abs(u.mean()) < 0.02
    n = oracle.decode_bf16(synth.bf16_operands(256, 64, 256, "normal", workload=1)[0])
    assert abs(n.mean()) < 0.02 and abs(n.std() - 1) < 0.02
    ns = oracle.decode_bf16(synth.bf16_operands(256, 64, 4096, "normal_scaled", workload=1)[0])
    assert abs(ns.std() * 64 - 1) < 0.02
    i = oracle.decode_bf16(synth.bf16_operands(64, 64, 256, "ints", workload=1)[0])
    assert set(np.unique(i)) == set(range(-4, 5))


def test_padding_columns_and_mxfp8_recipe():
    a, b = synth.bf16_operands(5, 6, 10, "uniform", workload=4, lda=16, ldb=24)
    assert a.shape == (5, 16) and b.shape == (6, 24)
    assert np.all(a[:, 10:] == 0x7FC0)
    a, sfa, b, sfb = synth.mxfp8_operands(8, 4, 64, workload=4)
    assert a.dtype == np.uint8 and sfa.shape == (8, 2) and sfb.shape == (4, 2)
    assert sfa.min() >= 123 and sfa.max() <= 131
    v = oracle.decode_e4m3(a)
    assert np.all(np.abs(v) <= 1)
