"""The FP8 quantiser divides by the block scale with a correctly rounded
reciprocal and two Markstein corrections instead of an IEEE division per
element.  This checks that quotient against CUDA's IEEE division: the E4M3
codes always agree, and the quotients agree bit for bit wherever
|x/s| >= 2^-12 (below that every code is +-0).  Every fp32 mantissa of x is
tried against thousands of scales, including scales whose reciprocal is
inexact by almost half an ulp, the all-ones mantissa, and the smallest scale
the fast path accepts (2^-90) with quotients near the smallest E4M3
magnitude and zero or subnormal x."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "cuda", "quotient_check.cu")


# both forms of the packed quotient: two Markstein corrections, and the
# two-term reciprocal with one correction
@pytest.fixture(scope="module", params=["two_corrections", "two_term_reciprocal"])
def qlib(request, tmp_path_factory):
    import torch
    assert torch.cuda.is_available()
    so = str(tmp_path_factory.mktemp("qcheck") / "libqcheck.so")
    form = ["-DRLX_QUOTIENT_2TERM=1"] if request.param == "two_term_reciprocal" else []
    subprocess.check_call(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-O3", "-std=c++20", "-fmad=false", "-Xcompiler", "-fPIC", "-shared",
                           *form, "-o", so, SRC])
    L = ctypes.CDLL(so)
    L.quotient_check.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_uint32, ctypes.c_uint32,
                                 ctypes.c_void_p, ctypes.c_void_p]
    L.quotient_check.restype = ctypes.c_int
    return L


def _check(L, scales, x_first, nx):
    s = np.ascontiguousarray(scales, dtype=np.float32)
    m = np.zeros(1, dtype=np.uint64)
    w = np.zeros(4, dtype=np.uint32)
    rc = L.quotient_check(s.ctypes.data, s.size, x_first, nx, m.ctypes.data, w.ctypes.data)
    assert rc == 0, "CUDA error %d" % rc
    assert m[0] == 0, "%d mismatches, e.g. x=%08x s=%08x fast=%08x ieee=%08x" % (m[0], *w)


def _scales(rng, k, exp_bits):
    mant = rng.integers(0, 1 << 23, size=k, dtype=np.uint32)
    special = np.array([0, 1, 2, 0x7FFFFF, 0x7FFFFE, 0x400000, 0x3FFFFF, 0x124925, 0x555555, 0x2AAAAA],
                       dtype=np.uint32)
    mant = np.concatenate([special, mant])
    return ((np.uint32(exp_bits) << 23) | mant).view(np.float32)


def test_quotient_all_mantissas(qlib):
    rng = np.random.default_rng(1234)
    s = _scales(rng, 2038, 127)                     # s in [1, 2)
    for x_exp in (127, 128, 134):                   # x in [1, 2), [2, 4), [128, 256)
        _check(qlib, s, x_exp << 23, 1 << 23)
        _check(qlib, s[:256], (x_exp << 23) | 0x80000000, 1 << 23)   # negative x


def test_quotient_reciprocal_rounding_extremes(qlib):
    """Scales whose reciprocal rounds by nearly half an ulp."""
    rng = np.random.default_rng(99)
    cand = _scales(rng, 1 << 20, 127).astype(np.float64)
    err = np.abs(1.0 / cand - (1.0 / cand).astype(np.float32).astype(np.float64)) * cand
    worst = cand[np.argsort(-err)[:512]].astype(np.float32)
    _check(qlib, worst, 127 << 23, 1 << 23)
    _check(qlib, worst, 128 << 23, 1 << 23)


def test_quotient_smallest_fast_scale(qlib):
    """s just above 2^-90: quotients from 2^-14 to 2^-8 (around the smallest
    E4M3 magnitudes) and zero / tiny x."""
    rng = np.random.default_rng(5)
    s = _scales(rng, 118, 127 - 90)                 # s in [2^-90, 2^-89)
    for q_exp in range(-14, -7):
        _check(qlib, s, (127 - 90 + q_exp) << 23, 1 << 23)
    _check(qlib, s, 0, 1 << 22)                     # +0 and the smallest subnormals
    _check(qlib, s, 0x80000000, 1 << 22)            # -0 and negative subnormals


def test_quotient_large_scale(qlib):
    rng = np.random.default_rng(6)
    s = _scales(rng, 118, 127 + 100)                # s near 2^100
    _check(qlib, s, (127 + 101) << 23, 1 << 23)
