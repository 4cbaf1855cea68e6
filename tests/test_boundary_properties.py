"""Property test of the C ABI's argument contract (include/b200gemm.h) on the
host: from a valid call, any single documented violation returns its
documented status, and nothing is launched.  Without a device the valid call
itself reports GEMM_ERR_UNSUPPORTED_DEVICE, so the whole test is skipped on
a machine with a GPU (a valid call there would launch on these fake pointers)."""
import pytest
import torch
from hypothesis import given, settings
from hypothesis import strategies as st

from dense_gemm_engineering_bf16_b200 import gemm as G

pytestmark = pytest.mark.skipif(torch.cuda.is_available(), reason="checks the host-side contract only")

BASE_A, BASE_B, BASE_C, BASE_BIAS = 0x7E0000000000, 0x7E4000000000, 0x7E8000000000, 0x7EC000000000
OK, INVALID, MISALIGNED, ALIAS, NO_DEVICE, TOO_LARGE = 0, 1, 2, 3, 4, 7


def up8(x):
    return x + (-x % 8)


@st.composite
def calls(draw):
    M, N, K = (draw(st.integers(1, 5000)) for _ in range(3))
    f32 = draw(st.booleans())
    a_mn, b_mn = draw(st.booleans()), draw(st.booleans())
    c = dict(A=BASE_A, B=BASE_B, C=BASE_C, M=M, N=N, K=K,
             lda=up8(M if a_mn else K) + 8 * draw(st.integers(0, 3)),
             ldb=up8(N if b_mn else K) + 8 * draw(st.integers(0, 3)),
             ldc=(N + (-N % 4) if f32 else up8(N)) + 8 * draw(st.integers(0, 3)),
             ct=G.OUT_F32 if f32 else G.OUT_BF16, al=int(a_mn), bl=int(b_mn),
             bias=draw(st.sampled_from([0, BASE_BIAS])), act=draw(st.integers(0, 3)))
    return c


def run(c):
    return G.lib.gemm_bf16_fused(c["A"], c["B"], c["C"], c["M"], c["N"], c["K"], c["lda"], c["ldb"], c["ldc"],
                                 c["ct"], c["al"], c["bl"], 1.0, 0.0, c["bias"], c["act"], 0)


MUTATIONS = {
    "negative M": (lambda c: c.update(M=-1), INVALID),
    "negative K": (lambda c: c.update(K=-3), INVALID),
    "bad c_type": (lambda c: c.update(ct=2), INVALID),
    "bad layout": (lambda c: c.update(al=2), INVALID),
    "bad act": (lambda c: c.update(act=4), INVALID),
    "ldc < N": (lambda c: c.update(ldc=c["N"] - 1), INVALID),
    "lda too small": (lambda c: c.update(lda=(c["M"] if c["al"] else c["K"]) - 1), INVALID),
    "ldb too small": (lambda c: c.update(ldb=(c["N"] if c["bl"] else c["K"]) - 1), INVALID),
    "null C": (lambda c: c.update(C=0), INVALID),
    "null A": (lambda c: c.update(A=0), INVALID),
    "A misaligned": (lambda c: c.update(A=c["A"] + 8), MISALIGNED),
    "C misaligned": (lambda c: c.update(C=c["C"] + 4), MISALIGNED),
    "bias misaligned": (lambda c: c.update(bias=BASE_BIAS + 4), MISALIGNED),
    "lda pitch": (lambda c: c.update(lda=c["lda"] + 1), MISALIGNED),
    "ldc pitch": (lambda c: c.update(ldc=c["ldc"] + 1), MISALIGNED),
    "C over A": (lambda c: c.update(C=c["A"]), ALIAS),
    "C over B": (lambda c: c.update(C=c["B"]), ALIAS),
    "bias in C": (lambda c: c.update(bias=c["C"]), ALIAS),
    "M too large": (lambda c: c.update(M=1 << 31), TOO_LARGE),
}


@settings(max_examples=300, deadline=None)
@given(calls(), st.sampled_from(sorted(MUTATIONS)))
def test_one_violation_gives_its_status(c, name):
    assert run(dict(c)) == NO_DEVICE                   # the unmutated call is valid
    mutate, want = MUTATIONS[name]
    bad = dict(c)
    mutate(bad)
    if name == "lda pitch" and bad["lda"] * 2 % 16 == 0:
        return
    if name == "ldc pitch" and bad["ldc"] * (4 if bad["ct"] == G.OUT_F32 else 2) % 16 == 0:
        return
    got = run(bad)
    assert got == want, (name, bad, got)


@settings(max_examples=100, deadline=None)
@given(calls())
def test_empty_problems_are_ok_without_checking_pointers(c):
    for dim in ("M", "N"):
        e = dict(c, A=0, B=0, C=0, bias=BASE_BIAS + 4)
        e[dim] = 0
        assert run(e) == OK
