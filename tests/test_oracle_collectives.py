"""Pins of the oracle's quantiser and collectives (CPU only).

Each test holds the oracle against something other than itself: the pages'
worked example, closed forms, exact rational sums, fp64/torch restatements
(tests/refpipe.py), the textbook error bound of recursive summation, and
invariants between collectives (flat == tree on a native wire, reduce-scatter
then all-gather == tree on the FP8 wire, alltoall is a chunk transpose).
"""
import os
from fractions import Fraction

import numpy as np
import pytest

import refpipe
from precision_collective_reduction_fp32_b200 import synth

HERE = os.path.dirname(os.path.abspath(__file__))
U = 2.0 ** -24   # unit roundoff of binary32


def _golden_worked_example():
    rows = []
    with open(os.path.join(HERE, "golden", "worked_example.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                n, a, b, e = line.split()
                rows.append((int(n), int(a) * int(b), float(e)))
    return rows


def _as_f32(x):
    return refpipe.bf16_to_f32(x) if x.dtype == np.uint16 else x


def _rows_wire(x32, wire_fp8, lo=0, hi=None):
    return [refpipe.wire(x32[s, lo:hi], wire_fp8) for s in range(x32.shape[0])]


# ------------------------------------------------------------ quantiser

@pytest.mark.parametrize("n", [1, 7, 127, 128, 129, 200, 1000, 4096 + 3])
@pytest.mark.parametrize("dist", ["normal", "normal_outliers", "student_t3"])
def test_quantize_matches_fp64_torch_restatement(orc, n, dist):
    x = synth.draw_row(dist, n, 11 + n)
    codes, scales = orc.quantize(x[None, :])
    c_ref, s_ref, d_ref = refpipe.quant_segment(x)
    assert refpipe.same_bits(codes[0], c_ref)
    assert refpipe.same_bits(scales[0].view(np.uint32), s_ref.view(np.uint32))
    y = orc.dequantize(codes, scales)
    assert refpipe.same_bits(y[0].view(np.uint32), d_ref.view(np.uint32))


def test_quantize_special_blocks(orc):
    """All-zero blocks (scale 0, signed zero codes), amax underflowing the scale,
    fp32 subnormal scales, partial last block."""
    x = np.zeros(5 * 128 + 17, dtype=np.float32)
    x[1] = -0.0
    x[128:256] = np.float32(1e-44) * np.sign(np.arange(128) - 63.5).astype(np.float32)  # s underflows to 0
    x[256:384] = np.float32(3e-37)       # subnormal scale 6.7e-40
    x[300] = -np.float32(3e-37)
    x[384:512] = np.linspace(-5, 5, 128, dtype=np.float32)
    x[640:] = np.float32(-2.5)
    codes, scales = orc.quantize(x[None, :])
    c_ref, s_ref, d_ref = refpipe.quant_segment(x)
    assert refpipe.same_bits(codes[0], c_ref) and refpipe.same_bits(scales[0], s_ref)
    assert scales[0, 0] == 0 and codes[0, 1] == 0x80 and codes[0, 0] == 0x00
    assert scales[0, 1] == 0 and np.array_equal(codes[0, 128:256] & 0x80, np.where(x[128:256] < 0, 0x80, 0))
    assert 0 < scales[0, 2] < np.finfo(np.float32).tiny          # subnormal scale
    assert codes[0, 256] == 0x7E and codes[0, 300] == 0xFE
    y = orc.dequantize(codes, scales)[0]
    assert refpipe.same_bits(y.view(np.uint32), d_ref.view(np.uint32))


def test_quantize_bf16_widens_exactly(orc):
    x = synth.as_bf16_bits(synth.draw_row("normal", 1000, 5))
    codes, scales = orc.quantize(x[None, :])
    c_ref, s_ref, _ = refpipe.quant_segment(refpipe.bf16_to_f32(x))
    assert refpipe.same_bits(codes[0], c_ref) and refpipe.same_bits(scales[0], s_ref)
    yb = orc.dequantize(codes, scales, dtype=np.uint16)[0]
    yf = orc.dequantize(codes, scales)[0]
    assert refpipe.same_bits(yb, refpipe.f32_to_bf16_torch(yf))


def test_quantize_error_bound(orc):
    """e4m3 keeps 3 mantissa bits: a normal-range code is within 2^-4 relative,
    a subnormal one within 2^-10 * s absolute; the amax element comes back
    within 2 ulp (its code is 448 or 448 rounded from just above)."""
    for dist in ("normal", "normal_outliers", "student_t3"):
        x = synth.draw_row(dist, 128 * 512, 99)
        codes, scales = orc.quantize(x[None, :])
        y = orc.dequantize(codes, scales)[0].astype(np.float64)
        s = np.repeat(scales[0].astype(np.float64), 128)
        err = np.abs(y - x)
        bound = np.maximum(2.0 ** -4 * np.abs(x), 2.0 ** -10 * s) * (1 + 2.0 ** -20) + 2 * U * np.abs(x)
        assert np.all(err <= bound)
        blocks = x.reshape(-1, 128)
        amax = np.abs(blocks).max(1)
        am_idx = np.abs(blocks).argmax(1)
        yb = y.reshape(-1, 128)[np.arange(blocks.shape[0]), am_idx]
        assert np.all(np.abs(np.abs(yb) - amax) <= 2 * np.spacing(amax.astype(np.float32)))


def test_quantize_rows_anchor_blocks_at_row_start(orc):
    x = synth.rank_buffers(1, count=300, nranks=3, stride=308)
    codes, scales = orc.quantize(x, n=300)
    for r in range(3):
        c_ref, s_ref, _ = refpipe.quant_segment(x[r, :300])
        assert refpipe.same_bits(codes[r, :300], c_ref) and refpipe.same_bits(scales[r], s_ref)


# ------------------------------------------------------- worked example

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("algo", ["flat", "tree"])
@pytest.mark.parametrize("wire", [0, 1])
def test_worked_example(orc, dtype, algo, wire):
    for nranks, count, expected in _golden_worked_example():
        x = synth.full_rank_values(nranks, count, dtype)
        fn = orc.allreduce_flat if algo == "flat" else orc.allreduce_tree
        y = _as_f32(fn(x, wire=wire))
        assert np.all(y == expected), (nranks, dtype, algo, wire)


def test_worked_example_fp8_payload_closed_form(orc):
    """Rank r's block is all r: scale = fl32(r/448), every code 0x7E (448), and
    448 * scale rounds back to exactly r.  The tree's second quantisation of
    the sum 28 has scale fl32(28/448) = 1/16 exactly."""
    x = synth.full_rank_values(8, 200)
    codes, scales = orc.quantize(x, n=200)
    for r in range(1, 8):
        assert np.all(codes[r] == 0x7E)
        assert scales[r, 0] == np.float32(r / 448.0) == scales[r, 1]
        assert np.float32(448.0 * np.float64(scales[r, 0])) == r
    assert np.all(codes[0] == 0) and np.all(scales[0] == 0)
    assert np.float32(28 / 448.0) == 0.0625


# ---------------------------------------------------- rank order, exact sums

def test_sum_is_rank_ordered(orc):
    """1 + 2^-24 + 2^-24 in rank order rounds twice to 1 (ties to even); the
    reversed order is exact.  Any other order or a pairwise tree breaks this."""
    x = np.array([[1.0], [2.0 ** -24], [2.0 ** -24]], dtype=np.float32)
    assert orc.allreduce_flat(x)[0, 0] == 1.0
    assert orc.allreduce_flat(x[::-1].copy())[0, 0] == np.float32(1 + 2.0 ** -23)
    assert orc.allreduce_tree(x)[2, 0] == 1.0


def test_bruteforce_tiny_exact_sums(orc):
    """N <= 3 ranks, count <= 3, values k * 2^e with small k: every fp32 sum is
    exact, so the result must equal the exact rational sum; on the FP8 wire
    values on the e4m3 grid times a power-of-two scale survive exactly."""
    rng = np.random.default_rng(0)
    for trial in range(300):
        nranks = int(rng.integers(1, 4))
        count = int(rng.integers(1, 4))
        k = rng.integers(-15, 16, size=(nranks, count))
        e = rng.integers(-4, 5, size=(nranks, count))
        x = (k * np.exp2(e)).astype(np.float32)
        exact = [sum(Fraction(float(x[s, i])) for s in range(nranks)) for i in range(count)]
        for fn in (orc.allreduce_flat, orc.allreduce_tree):
            y = fn(x)
            assert all(Fraction(float(y[r, i])) == exact[i] for r in range(nranks) for i in range(count))
        # FP8 wire: make every row's block amax 448 * 2^g so the scale is 2^g and
        # every value (e4m3 grid) * 2^g quantises without error.
        g = int(rng.integers(-6, 6))
        grid = np.array([orc.e4m3_value(c) for c in range(0x7F)], dtype=np.float64)
        vals = rng.choice(grid, size=(nranks, count)) * np.where(rng.random((nranks, count)) < .5, -1, 1)
        vals[:, 0] = 448.0
        xf = (vals * 2.0 ** g).astype(np.float32)
        exact = [sum(Fraction(float(xf[s, i])) for s in range(nranks)) for i in range(count)]
        y = orc.allreduce_flat(xf, wire=1)
        for i in range(count):
            if Fraction(float(np.float32(float(exact[i])))) == exact[i]:
                assert Fraction(float(y[0, i])) == exact[i]


def test_recursive_sum_error_bound(orc):
    """|fl32 sum - exact| <= (N-1) u sum|x| (Higham, recursive summation)."""
    for n in (2, 3, 8, 16):
        x = synth.rank_buffers(4, count=4096, nranks=n)
        y = orc.allreduce_flat(x)[0].astype(np.float64)
        exact = x.astype(np.float64).sum(0)
        bound = (n - 1) * U * np.abs(x).astype(np.float64).sum(0) * (1 + 1e-6)
        assert np.all(np.abs(y - exact) <= bound)


# ----------------------------------------------------- flat and tree vs restatement

CASES = [(n, c) for n in (2, 3, 4, 8) for c in (1, 7, 127, 128, 129, 200, 1000, 3 * 128 * 8 + 5)]


@pytest.mark.parametrize("nranks,count", CASES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_flat_matches_restatement(orc, nranks, count, dtype):
    x = synth.rank_buffers(4, count=count, nranks=nranks, stride=count + 3, dtype=dtype)
    x32 = _as_f32(x)
    for wire in (0, 1):
        y = orc.allreduce_flat(x, wire=wire, count=count)
        ref = refpipe.ordered_sum(_rows_wire(x32, wire, 0, count))
        if dtype == "bf16":
            ref = refpipe.f32_to_bf16_torch(ref)
        for r in range(nranks):
            assert refpipe.same_bits(y[r, :count], ref), (wire, r)
            assert not y[r, count:].any()  # padding untouched (zeros in the fresh output)


@pytest.mark.parametrize("nranks,count", CASES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_tree_matches_restatement(orc, nranks, count, dtype):
    x = synth.rank_buffers(5, count=count, nranks=nranks, dtype=dtype)
    x32 = _as_f32(x)
    flat = orc.allreduce_flat(x)
    assert refpipe.same_bits(orc.allreduce_tree(x), flat)           # native: tree == flat, bitwise
    y = orc.allreduce_tree(x, wire=1)
    s = refpipe.ordered_sum(_rows_wire(x32, True))
    ref = refpipe.quant_segment(s)[2]                             # second quantisation
    if dtype == "bf16":
        ref = refpipe.f32_to_bf16_torch(ref)
    for r in range(nranks):
        assert refpipe.same_bits(y[r], ref)


def test_tree_chunking(orc):
    assert orc.tree_chunk(200, 8) == 128
    assert orc.tree_chunk(16_777_216, 8) == 2_097_152
    assert orc.tree_chunk(33_554_432, 8) == 4_194_304
    assert orc.tree_chunk(1, 4) == 128
    assert orc.tree_chunk(129 * 128, 8) == 17 * 128


def test_inplace_allreduce(orc):
    x = synth.rank_buffers(4, count=1000, nranks=8)
    for fn in (orc.allreduce_flat, orc.allreduce_tree):
        for wire in (0, 1):
            ref = fn(x, wire=wire)
            z = x.copy()
            fn(z, wire=wire, out=z)
            assert refpipe.same_bits(z, ref)


def test_one_rank_is_identity(orc):
    for dtype in ("f32", "bf16"):
        x = synth.rank_buffers(5, count=300, nranks=1, dtype=dtype)
        for wire in (0, 1):
            assert refpipe.same_bits(orc.allreduce_flat(x, wire=wire), x)
            assert refpipe.same_bits(orc.allreduce_tree(x, wire=wire), x)
            assert refpipe.same_bits(orc.reduce_scatter(x, 300, wire=wire), x)
            assert refpipe.same_bits(orc.all_gather(x, 300, wire=wire), x)
            assert refpipe.same_bits(orc.alltoall(x, 300, wire=wire), x)


# ------------------------------------------------------- RS / AG / alltoall

@pytest.mark.parametrize("nranks,m", [(2, 1), (3, 7), (4, 128), (8, 129), (8, 256), (5, 300)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_reduce_scatter(orc, nranks, m, dtype):
    x = synth.rank_buffers(5, count=nranks * m, nranks=nranks, dtype=dtype)
    x32 = _as_f32(x)
    for wire in (0, 1):
        y = orc.reduce_scatter(x, m, wire=wire)
        for r in range(nranks):
            ref = refpipe.ordered_sum(_rows_wire(x32, wire, r * m, (r + 1) * m))
            if dtype == "bf16":
                ref = refpipe.f32_to_bf16_torch(ref)
            assert refpipe.same_bits(y[r], ref)


@pytest.mark.parametrize("nranks,m", [(2, 1), (3, 7), (4, 128), (8, 129), (5, 300)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_all_gather(orc, nranks, m, dtype):
    x = synth.rank_buffers(5, count=m, nranks=nranks, dtype=dtype)
    assert refpipe.same_bits(orc.all_gather(x, m), np.tile(x.reshape(1, -1), (nranks, 1)))
    y = orc.all_gather(x, m, wire=1)
    x32 = _as_f32(x)
    row = np.concatenate(_rows_wire(x32, True))
    if dtype == "bf16":
        row = refpipe.f32_to_bf16_torch(row)
    assert refpipe.same_bits(y, np.tile(row[None, :], (nranks, 1)))


@pytest.mark.parametrize("nranks,m", [(2, 1), (3, 7), (4, 128), (8, 129), (5, 300)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_alltoall_is_chunk_transpose(orc, nranks, m, dtype):
    x = synth.rank_buffers(5, count=nranks * m, nranks=nranks, dtype=dtype)
    y = orc.alltoall(x, m)
    t = x.reshape(nranks, nranks, m).transpose(1, 0, 2).reshape(nranks, nranks * m)
    assert refpipe.same_bits(y, t)
    assert refpipe.same_bits(orc.alltoall(y, m), x)                     # involution
    assert np.array_equal(np.sort(y.ravel()), np.sort(x.ravel()))   # a permutation
    yq = orc.alltoall(x, m, wire=1)
    x32 = _as_f32(x)
    for r in range(nranks):
        for s in range(nranks):
            ref = refpipe.wire(x32[s, r * m:(r + 1) * m], True)
            if dtype == "bf16":
                ref = refpipe.f32_to_bf16_torch(ref)
            assert refpipe.same_bits(yq[r, s * m:(s + 1) * m], ref)


@pytest.mark.parametrize("nranks,m", [(2, 128), (4, 256), (8, 384)])
def test_rs_then_ag_equals_tree_fp8(orc, nranks, m):
    """With block-aligned chunks, reduce-scatter (one quantisation) followed by
    all-gather (the second) is the FP8 tree allreduce, bit for bit."""
    x = synth.rank_buffers(4, count=nranks * m, nranks=nranks)
    rs = orc.reduce_scatter(x, m, wire=1)
    ag = orc.all_gather(rs, m, wire=1)
    assert refpipe.same_bits(ag, orc.allreduce_tree(x, wire=1))
    rs0 = orc.reduce_scatter(x, m)
    assert refpipe.same_bits(orc.all_gather(rs0, m), orc.allreduce_flat(x))


def test_fp8_wire_rejects_nonfinite(orc):
    x = np.ones((2, 130), dtype=np.float32)
    x[1, 5] = np.inf
    with pytest.raises(ValueError):
        orc.allreduce_flat(x, wire=1)
    orc.allreduce_flat(x, wire=0)   # a native wire just adds


def test_signed_zero_survives_the_sum(orc):
    """IEEE: (-0) + (-0) = -0.  Summing from the first term keeps it; a sum
    started from +0 would not.  On the FP8 wire -0 has code 0x80, scale 0."""
    x = np.full((3, 130), -0.0, dtype=np.float32)
    for fn in (orc.allreduce_flat, orc.allreduce_tree):
        for wire in (0, 1):
            y = fn(x, wire=wire)
            assert np.all(y.view(np.uint32) == 0x80000000), (fn, wire)
    codes, scales = orc.quantize(x)
    assert np.all(codes == 0x80) and np.all(scales == 0)
