"""E4M3 codes where the quotient's rounding decides them, against the oracle.

Blocks are built so that their quotients x/s fall on, and within a few fp32
ulps of, every E4M3 rounding boundary (fp32 input: 14 % of the quotients are
ties, and in 27 % the one-multiply estimate x * fl32(1/s) differs from the
correctly rounded quotient), and every bf16 bit pattern is tried (bf16
input); codes, scales and the FP8 DDA-flat and DDA-tree results must match
the oracle bit for bit.  Two builds run the same calls: the product, and the
profiling build RLX_QUOTIENT=3, which forms each block's codes from two
products that bracket the correctly rounded quotient and takes the full
quotient only for blocks where the two products' codes differ.
"""
import numpy as np
import pytest
import torch

import oracle
import refpipe
from gpuutil import stream, to_dev, to_host
from precision_collective_reduction_fp32_b200 import binding as B
from precision_collective_reduction_fp32_b200 import build as rlx_build
from test_gpu_bf16_special import _special_rows

pytestmark = pytest.mark.gpu

FP8 = B.RLX_WIRE_FP8_E4M3


# the product build (correctly rounded quotient by Markstein corrections) and
# the bracketing profiling build, through the same calls
@pytest.fixture(scope="module", params=["product", "bracket_quotient"])
def blib(request):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    oracle.build()
    if request.param == "product":
        rlx_build.build()
        return B.lib()
    return B.load(rlx_build.build_variant(request.param))


def _midpoint_rows(n=8, nblk=2048, seed=77):
    """[n, nblk*128] fp32: element 0 of each block is its amax A; the others
    are fl32(M * s) moved by -3..3 ulps, s = fl32(A / 448), M an E4M3
    rounding boundary (the midpoint of two neighbouring magnitudes)."""
    rng = np.random.default_rng(seed)
    mags = np.array([oracle.e4m3_value(c) for c in range(127)], dtype=np.float64)
    mids = ((mags[:-1] + mags[1:]) / 2).astype(np.float32)      # exact in fp32
    x = np.empty((n, nblk, 128), dtype=np.float32)
    amax = (rng.uniform(0.5, 2.0, size=(n, nblk)) *
            2.0 ** rng.integers(-20, 20, size=(n, nblk))).astype(np.float32)
    s = amax / np.float32(448.0)                                  # fl32(A / 448)
    m = mids[rng.integers(0, mids.size, size=(n, nblk, 127))]
    v = m * s[:, :, None]                                         # fl32(M * s)
    steps = rng.integers(-3, 4, size=v.shape)
    for k in range(1, 4):
        up, dn = steps >= k, steps <= -k
        v[up] = np.nextafter(v[up], np.float32(np.inf))
        v[dn] = np.nextafter(v[dn], np.float32(0))
    v *= np.where(rng.random(v.shape) < 0.5, -1, 1).astype(np.float32)
    x[:, :, 0] = amax
    x[:, :, 1:] = v
    return x.reshape(n, nblk * 128)


def _run(L, x):
    n, count = x.shape
    dc = B.RLX_BF16 if x.dtype == np.uint16 else B.RLX_F32
    dx = to_dev(x)
    codes = torch.empty((n, count), dtype=torch.uint8, device="cuda")
    scales = torch.empty((n, count // 128), dtype=torch.float32, device="cuda")
    flat, tree = torch.empty_like(dx), torch.empty_like(dx)
    wsb = B.rlx_workspace_bytes(B.RLX_COLL_ALLREDUCE_TREE, count, n, dc, FP8)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    assert L.rlx_quantize_fp8(dx.data_ptr(), dc, n, count, count, codes.data_ptr(),
                              scales.data_ptr(), stream()) == B.RLX_OK
    assert L.rlx_allreduce_flat(dx.data_ptr(), flat.data_ptr(), count, count, n, dc, FP8,
                                B.RLX_SUM, stream()) == B.RLX_OK
    assert L.rlx_allreduce_tree(dx.data_ptr(), tree.data_ptr(), count, count, n, dc, FP8,
                                B.RLX_SUM, ws.data_ptr(), wsb, stream()) == B.RLX_OK
    torch.cuda.synchronize()
    return to_host(codes), to_host(scales), to_host(flat), to_host(tree)


def _compare(x, got):
    codes, scales, flat, tree = got
    oc, os_ = oracle.quantize(x)
    assert np.array_equal(codes, oc), "codes: %d differ" % int((codes != oc).sum())
    assert refpipe.same_bits(scales, os_), "scales"
    assert refpipe.same_bits(flat, oracle.allreduce_flat(x, wire=oracle.FP8)), "DDA-flat"
    assert refpipe.same_bits(tree, oracle.allreduce_tree(x, wire=oracle.FP8)), "DDA-tree"


def test_bracket_codes_at_rounding_boundaries(blib):
    x = _midpoint_rows()
    _compare(x, _run(blib, x))


def test_bracket_codes_every_bf16_pattern(blib):
    x = _special_rows()
    _compare(x, _run(blib, x))
