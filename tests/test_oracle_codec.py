"""Pins of the oracle's e4m3 and bf16 codecs (CPU only).

The oracle encodes with integer bit arithmetic; these tests hold it against
(a) facts of the OCP FP8 E4M3 format, (b) torch's float8_e4m3fn and bfloat16
conversions (library routines, round-to-nearest-even), and (c) a brute-force
nearest-value search over the 127 finite non-negative e4m3 magnitudes with
ties to the even code.
"""
import math

import numpy as np
import pytest

import refpipe


def test_decode_ocp_facts(orc):
    assert orc.e4m3_value(0x7E) == 448.0          # largest finite
    assert orc.e4m3_value(0xFE) == -448.0
    assert orc.e4m3_value(0x08) == 2.0 ** -6      # smallest normal
    assert orc.e4m3_value(0x01) == 2.0 ** -9      # smallest subnormal
    assert orc.e4m3_value(0x07) == 7 * 2.0 ** -9  # largest subnormal
    assert orc.e4m3_value(0x38) == 1.0
    assert orc.e4m3_value(0x00) == 0.0 and math.copysign(1, orc.e4m3_value(0x80)) == -1
    assert math.isnan(orc.e4m3_value(0x7F)) and math.isnan(orc.e4m3_value(0xFF))


def test_decode_all_codes_vs_torch(orc):
    codes = np.arange(256, dtype=np.uint8)
    mine = np.array([orc.e4m3_value(c) for c in codes], dtype=np.float32)
    ref = refpipe.e4m3_decode_torch(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def _finite_magnitudes():
    v = np.array([np.float64(np.float32(refpipe.e4m3_decode_torch(np.array([c], np.uint8))[0]))
                  for c in range(0x7F)])
    return v  # codes 0x00..0x7E, increasing


def _bruteforce_encode(x: np.ndarray) -> np.ndarray:
    """Nearest of the 127 magnitudes by explicit midpoint search, ties to even code,
    |x| >= 448 saturating.  Midpoints of neighbouring e4m3 values are exact in fp64."""
    mags = _finite_magnitudes()
    ax = np.abs(x.astype(np.float64))
    out = np.empty(x.shape, dtype=np.uint8)
    for i, a in enumerate(ax):
        if a >= 448.0:
            k = 0x7E
        else:
            k = int(np.searchsorted(mags, a, side="right")) - 1  # mags[k] <= a < mags[k+1]
            if mags[k] != a:
                mid = (mags[k] + mags[k + 1]) / 2
                if a > mid or (a == mid and (k & 1)):
                    k += 1
        out[i] = k | (0x80 if np.signbit(x[i]) else 0)
    return out


def test_encode_ties_and_neighbours_bruteforce(orc):
    mags = _finite_magnitudes()
    pts = []
    for k in range(0x7E):
        mid = np.float32((mags[k] + mags[k + 1]) / 2)
        pts += [mags[k], mid, np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(1e9))]
    pts += [448.0, np.nextafter(np.float32(448), np.float32(0)), 448.5, 464.0, 1e30,
            np.finfo(np.float32).max, 2.0 ** -10, 2.0 ** -11, 1e-45, 0.0]
    x = np.array(pts, dtype=np.float32)
    x = np.concatenate([x, -x])
    mine = np.array([orc.e4m3_encode(v) for v in x], dtype=np.uint8)
    assert np.array_equal(mine, _bruteforce_encode(x))


def test_encode_random_bruteforce(orc):
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 0x7F800000, size=20000, dtype=np.uint32)   # finite magnitudes
    x = bits.view(np.float32) * np.where(rng.random(20000) < 0.5, -1, 1).astype(np.float32)
    near = (rng.standard_normal(20000) * 50).astype(np.float32)
    x = np.concatenate([x, near])
    mine = np.array([orc.e4m3_encode(v) for v in x], dtype=np.uint8)
    assert np.array_equal(mine, _bruteforce_encode(x))


def test_encode_exhaustive_band_vs_torch(orc):
    """Every fp32 magnitude from 2^-12 up to (not incl.) 464, both signs, against
    torch's round-to-nearest-even conversion; below 2^-12 everything is +-0."""
    lo, hi = 0x39800000, 0x43E80000        # 2^-12 .. 464
    step = 1 << 24
    for first in range(lo, hi, step):
        n = min(step, hi - first)
        mine = orc.e4m3_encode_bits_range(first, n)
        vals = np.arange(first, first + n, dtype=np.uint32).view(np.float32)
        assert np.array_equal(mine, refpipe.e4m3_encode_torch(vals)), hex(first)
        neg = orc.e4m3_encode_bits_range(first | 0x80000000, n)
        assert np.array_equal(neg, mine | 0x80), hex(first)
    small = orc.e4m3_encode_bits_range(0, lo)[:: 997]
    assert not small.any()
    assert np.all(orc.e4m3_encode_bits_range(0x80000000, 1 << 20) == 0x80)


def test_encode_saturates(orc):
    for v in (448.0, 449.0, 463.9, 464.0, 480.0, 1e6, 3.4e38):
        assert orc.e4m3_encode(v) == 0x7E
        assert orc.e4m3_encode(-v) == 0xFE
    for first in range(0x43E00000, 0x7F800000, 1 << 22):
        assert np.all(orc.e4m3_encode_bits_range(first, 1 << 14) == 0x7E), hex(first)


def test_bf16_rne_vs_torch(orc):
    rng = np.random.default_rng(3)
    x = rng.standard_normal(4000).astype(np.float32) * 1000
    ties = (rng.integers(0, 1 << 16, 2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    x = np.concatenate([x, ties, -ties, np.float32([0.0, -0.0, 1.0, 3.0e38, 1e-40])])
    x = x[np.isfinite(x)]
    mine = orc.f32_to_bf16(x)
    assert np.array_equal(mine, refpipe.f32_to_bf16_torch(x))
