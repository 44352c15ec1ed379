"""bf16 rank buffers holding every finite bf16 magnitude class the FP8 wire
can meet, through every FP8-wire collective, against the oracle bit for bit.

The reducing kernels find a bf16 block's amax in bf16x2 max arithmetic and
the others on widened fp32 values; both must keep subnormals (a flushed
subnormal amax would give a zero scale).  Seeded N(0,1) data never reaches
the bf16 subnormals, so here each of the 8 ranks holds its own permutation
of every bf16 bit pattern with |x| < 2^124 (both signs; small enough that no
fp32 sum of 8 ranks can overflow), followed by blocks made only of
subnormals (the largest subnormal, the smallest, all of them), blocks of
signed zeros, and blocks whose amax is the smallest normal.  Every output
element of DDA-flat, DDA-tree (two launches and one), reduce-scatter,
all-gather, alltoall and quantise/dequantise is compared with the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import refpipe
from gpuutil import stream, to_dev, to_host
from precision_collective_reduction_fp32_b200 import binding as B
from precision_collective_reduction_fp32_b200 import build as rlx_build

pytestmark = pytest.mark.gpu

N = 8
FP8 = B.RLX_WIRE_FP8_E4M3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    rlx_build.build()
    oracle.build()


def _special_rows():
    """[8, count] uint16 bf16 bit patterns; count a multiple of 8 * 128."""
    mags = np.arange(0, 0xFB << 7, dtype=np.uint16)            # exponent field < 0xFB
    pats = np.concatenate([mags, mags | 0x8000])               # both signs
    rng = np.random.default_rng(2024)
    tail = []
    sub = np.arange(1, 0x80, dtype=np.uint16)                  # every bf16 subnormal magnitude
    tail.append(np.resize(sub, 128))                            # amax: the largest subnormal
    tail.append(np.resize(sub, 128) | 0x8000)                   # the same, negative
    tail.append(np.full(128, 0x0001, np.uint16))                # amax: the smallest subnormal
    one = np.zeros(128, np.uint16); one[17] = 0x8001; tail.append(one)
    z = np.zeros(128, np.uint16); z[::3] = 0x8000; tail.append(z)   # signed zeros only
    tail.append(np.full(128, 0x8000, np.uint16))                # all -0
    mix = np.resize(sub, 128).copy(); mix[5] = 0x0080; tail.append(mix)  # smallest normal on top
    tail = np.concatenate(tail)
    rows = []
    for r in range(N):
        body = rng.permutation(pats)
        row = np.concatenate([body, np.roll(tail, 128 * r)])
        rows.append(row)
    count = len(rows[0])
    pad = (-count) % (N * 128)
    rows = [np.concatenate([row, np.zeros(pad, np.uint16)]) for row in rows]
    return np.stack(rows)


@pytest.fixture(scope="module")
def special():
    x = _special_rows()
    return x, to_dev(x)


def _same(a, b, what):
    assert refpipe.same_bits(a, b), what


def test_bf16_special_allreduces(special):
    x, dx = special
    n, count = x.shape
    out = torch.empty_like(dx)
    assert B.lib().rlx_allreduce_flat(dx.data_ptr(), out.data_ptr(), count, count, n, B.RLX_BF16,
                                      FP8, B.RLX_SUM, stream()) == B.RLX_OK
    torch.cuda.synchronize()
    _same(to_host(out), oracle.allreduce_flat(x, wire=oracle.FP8), "flat")
    ref_tree = oracle.allreduce_tree(x, wire=oracle.FP8)
    need = B.rlx_workspace_bytes(B.RLX_COLL_ALLREDUCE_TREE, count, n, B.RLX_BF16, FP8)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    assert B.lib().rlx_allreduce_tree(dx.data_ptr(), out.data_ptr(), count, count, n, B.RLX_BF16,
                                      FP8, B.RLX_SUM, ws.data_ptr(), need, stream()) == B.RLX_OK
    torch.cuda.synchronize()
    _same(to_host(out), ref_tree, "tree")
    need = B.rlx_workspace_bytes(B.RLX_COLL_ALLREDUCE_TREE_FUSED, count, n, B.RLX_BF16, FP8)
    fws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    out.zero_()
    assert B.lib().rlx_allreduce_tree_fused(dx.data_ptr(), out.data_ptr(), count, count, n,
                                            B.RLX_BF16, FP8, B.RLX_SUM, fws.data_ptr(), need,
                                            st.data_ptr(), 0, stream()) == B.RLX_OK
    torch.cuda.synchronize()
    assert int(st.item()) == B.RLX_OK
    _same(to_host(out), ref_tree, "tree_fused")


def test_bf16_special_chunked(special):
    x, dx = special
    n, count = x.shape
    m = count // n
    rs = torch.empty((n, m), dtype=torch.bfloat16, device="cuda")
    ag = torch.empty_like(dx)
    a2a = torch.empty_like(dx)
    assert B.lib().rlx_reduce_scatter(dx.data_ptr(), count, rs.data_ptr(), m, m, n, B.RLX_BF16,
                                      FP8, B.RLX_SUM, stream()) == B.RLX_OK
    assert B.lib().rlx_all_gather(rs.data_ptr(), m, ag.data_ptr(), count, m, n, B.RLX_BF16, FP8,
                                  stream()) == B.RLX_OK
    assert B.lib().rlx_alltoall(dx.data_ptr(), count, a2a.data_ptr(), count, m, n, B.RLX_BF16,
                                FP8, stream()) == B.RLX_OK
    torch.cuda.synchronize()
    ref_rs = oracle.reduce_scatter(x, m, wire=oracle.FP8)
    _same(to_host(rs), ref_rs, "reduce_scatter")
    _same(to_host(ag), oracle.all_gather(ref_rs, m, wire=oracle.FP8), "all_gather")
    _same(to_host(a2a), oracle.alltoall(x, m, wire=oracle.FP8), "alltoall")


def test_bf16_special_quantize(special):
    x, dx = special
    n, count = x.shape
    codes = torch.empty((n, count), dtype=torch.uint8, device="cuda")
    scales = torch.empty((n, count // 128), dtype=torch.float32, device="cuda")
    y = torch.empty_like(dx)
    assert B.lib().rlx_quantize_fp8(dx.data_ptr(), B.RLX_BF16, n, count, count, codes.data_ptr(),
                                    scales.data_ptr(), stream()) == B.RLX_OK
    assert B.lib().rlx_dequantize_fp8(codes.data_ptr(), scales.data_ptr(), n, count, count,
                                      y.data_ptr(), B.RLX_BF16, stream()) == B.RLX_OK
    torch.cuda.synchronize()
    oc, os_ = oracle.quantize(x)
    _same(to_host(codes), oc, "codes")
    _same(to_host(scales), os_, "scales")
    _same(to_host(y), oracle.dequantize(oc, os_, dtype=np.uint16), "dequantize")
    # the subnormal-only blocks really have nonzero, subnormal-range scales
    s = to_host(scales)
    assert (s[(s > 0) & (s < 2.0 ** -126)]).size > 0
