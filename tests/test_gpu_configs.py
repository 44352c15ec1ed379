"""GPU parity at the benchmark sizes, in the layout the benchmark uses.

The five workloads (see precision_collective_reduction_fp32_b200.synth) run
through the C ABI on contiguous [N][count] rank rows, and EVERY output
element is compared bit for bit with the CPU oracle run on the same host
bytes: allreduce (flat and tree, both wires), quantise codes and scales,
dequantise, reduce-scatter, all-gather and alltoall.  The oracle does one of
these operations on 8 x 64 MiB in a few seconds on one host core, 8 x 256 MiB
in well under a minute.

On top of the element-wise comparison, properties that hold at any size are
checked on the GPU: every rank's allreduce result is identical, DDA-tree ==
DDA-flat on the native wire, reduce-scatter then all-gather == DDA-tree on
the FP8 wire, alltoall undoes itself, and the FP8 results stay within the
e4m3 error bound of the exact (fp64) sum.
Bar: bit-exact everywhere.
"""
import numpy as np
import pytest
import torch

import oracle
from gpuutil import stream, to_dev, to_host
from precision_collective_reduction_fp32_b200 import binding as B
from precision_collective_reduction_fp32_b200 import build as rlx_build
from precision_collective_reduction_fp32_b200 import synth

pytestmark = pytest.mark.gpu

NAT, FP8 = B.RLX_WIRE_NATIVE, B.RLX_WIRE_FP8_E4M3
ORC = {NAT: oracle.NATIVE, FP8: oracle.FP8}
WNAME = {NAT: "native", FP8: "fp8"}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    rlx_build.build()
    oracle.build()


def assert_same(got, ref, what):
    """Bitwise equality of two host arrays; on failure name the first
    differing element and how many differ."""
    got, ref = np.ascontiguousarray(got), np.ascontiguousarray(ref)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    u = {1: np.uint8, 2: np.uint16, 4: np.uint32}[got.dtype.itemsize]
    g, r = got.view(u), ref.view(u)
    if np.array_equal(g, r):
        return
    bad = np.flatnonzero(g.ravel() != r.ravel())
    i = np.unravel_index(bad[0], got.shape)
    pytest.fail("%s: %d of %d elements differ; first at %s: got %r (0x%x), oracle %r (0x%x)"
                % (what, bad.size, got.size, i, got[i], int(g[i]), ref[i], int(r[i])))


def _allreduce(algo, dx, count, wire, dcode):
    n = dx.shape[0]
    out = torch.empty_like(dx)
    if algo == "flat":
        st = B.lib().rlx_allreduce_flat(dx.data_ptr(), out.data_ptr(), count, count, n, dcode,
                                        wire, B.RLX_SUM, stream())
    else:
        need = B.rlx_workspace_bytes(B.RLX_COLL_ALLREDUCE_TREE, count, n, dcode, wire)
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
        st = B.lib().rlx_allreduce_tree(dx.data_ptr(), out.data_ptr(), count, count, n, dcode,
                                        wire, B.RLX_SUM, ws.data_ptr(), need, stream())
    assert st == B.RLX_OK
    torch.cuda.synchronize()
    return out


def _rows_identical(out):
    flat = out.view(out.shape[0], -1)
    it = torch.int16 if flat.dtype == torch.bfloat16 else torch.int32
    return all(torch.equal(flat[0].view(it), flat[r].view(it)) for r in range(1, flat.shape[0]))


def _chunked(dx, dcode, wire):
    """reduce-scatter of dx, all-gather of its result and alltoall of dx,
    as the benchmark issues them."""
    n, count = dx.shape
    m = count // n
    rs = torch.empty((n, m), dtype=dx.dtype, device="cuda")
    ag = torch.empty_like(dx)
    a2a = torch.empty_like(dx)
    assert B.lib().rlx_reduce_scatter(dx.data_ptr(), count, rs.data_ptr(), m, m, n, dcode, wire,
                                      B.RLX_SUM, stream()) == B.RLX_OK
    assert B.lib().rlx_all_gather(rs.data_ptr(), m, ag.data_ptr(), count, m, n, dcode, wire,
                                  stream()) == B.RLX_OK
    assert B.lib().rlx_alltoall(dx.data_ptr(), count, a2a.data_ptr(), count, m, n, dcode, wire,
                                stream()) == B.RLX_OK
    torch.cuda.synchronize()
    return rs, ag, a2a


def _check_chunked_whole(x, dx, dcode, wire, tag):
    n, count = x.shape
    m = count // n
    rs, ag, a2a = _chunked(dx, dcode, wire)
    ref_rs = oracle.reduce_scatter(x, m, wire=ORC[wire])
    got_rs = to_host(rs)
    assert_same(got_rs, ref_rs, "%s reduce_scatter %s" % (tag, WNAME[wire]))
    del rs
    assert_same(to_host(ag), oracle.all_gather(ref_rs, m, wire=ORC[wire]),
                "%s all_gather %s" % (tag, WNAME[wire]))
    assert_same(to_host(a2a), oracle.alltoall(x, m, wire=ORC[wire]),
                "%s alltoall %s" % (tag, WNAME[wire]))
    return ag, a2a


# ---------------------------------------------------------------- workload 1

@pytest.mark.parametrize("algo", ["flat", "tree"])
@pytest.mark.parametrize("wire", [NAT, FP8])
def test_workload1_tiny_full_compare(algo, wire):
    """N=8, fp32 [10,20]: the whole output against the oracle."""
    x = synth.rank_buffers(1)
    out = _allreduce(algo, to_dev(x), 200, wire, B.RLX_F32)
    fn = oracle.allreduce_flat if algo == "flat" else oracle.allreduce_tree
    assert_same(to_host(out), fn(x, wire=ORC[wire]), "tiny %s %s" % (algo, WNAME[wire]))


# ---------------------------------------------------------------- workload 2

@pytest.mark.parametrize("algo", ["flat", "tree"])
@pytest.mark.parametrize("wire", [NAT, FP8])
def test_workload2_decode_full_compare(algo, wire):
    """N=8, bf16 [32, 8192]: fp32 accumulation, bf16 out; whole output."""
    x = synth.rank_buffers(2)
    out = _allreduce(algo, to_dev(x), x.shape[1], wire, B.RLX_BF16)
    fn = oracle.allreduce_flat if algo == "flat" else oracle.allreduce_tree
    assert_same(to_host(out), fn(x, wire=ORC[wire]), "decode %s %s" % (algo, WNAME[wire]))


# ---------------------------------------------------------------- workload 3

@pytest.fixture(scope="module")
def prefill():
    x = synth.rank_buffers(3)
    return x, to_dev(x)


@pytest.mark.parametrize("wire", [NAT, FP8])
def test_workload3_prefill_allreduce(prefill, wire):
    """N=8, bf16 [4096, 8192] (64 MiB/rank): DDA-tree and DDA-flat, whole
    output against the oracle; all rows identical; tree == flat (native)."""
    x, dx = prefill
    count = x.shape[1]
    tree = _allreduce("tree", dx, count, wire, B.RLX_BF16)
    assert_same(to_host(tree), oracle.allreduce_tree(x, wire=ORC[wire]),
                "prefill tree %s" % WNAME[wire])
    assert _rows_identical(tree)
    flat = _allreduce("flat", dx, count, wire, B.RLX_BF16)
    assert_same(to_host(flat), oracle.allreduce_flat(x, wire=ORC[wire]),
                "prefill flat %s" % WNAME[wire])
    if wire == NAT:
        assert torch.equal(tree.view(torch.int16), flat.view(torch.int16))


@pytest.mark.parametrize("wire", [NAT, FP8])
def test_workload3_prefill_chunked(prefill, wire):
    """The benchmark's bf16 reduce-scatter, all-gather and alltoall on the
    prefill rank buffers (m = 4 Mi elements): whole outputs."""
    x, dx = prefill
    _check_chunked_whole(x, dx, B.RLX_BF16, wire, "prefill")


# ---------------------------------------------------------------- workload 4

@pytest.fixture(scope="module")
def lp_allreduce():
    x = synth.rank_buffers(4)
    return x, to_dev(x)


@pytest.mark.parametrize("algo", ["tree", "flat"])
@pytest.mark.parametrize("wire", [FP8, NAT])
def test_workload4_lp_allreduce_whole(lp_allreduce, algo, wire):
    """N=8, fp32 [16,777,216] with 1% x100 outliers: DDA-tree (FP8: the
    fused dequantise-sum-requantise pass and the all-gather pass) and
    DDA-flat, every element of every rank against the oracle."""
    x, dx = lp_allreduce
    out = _allreduce(algo, dx, x.shape[1], wire, B.RLX_F32)
    fn = oracle.allreduce_flat if algo == "flat" else oracle.allreduce_tree
    assert_same(to_host(out), fn(x, wire=ORC[wire]), "lp-allreduce %s %s" % (algo, WNAME[wire]))
    assert _rows_identical(out)


def test_workload4_quantize_dequantize_whole(lp_allreduce):
    """rlx_quantize_fp8 / rlx_dequantize_fp8 over the whole batch: every
    code, every scale and every dequantised value against the oracle."""
    x, dx = lp_allreduce
    n, count = x.shape
    codes = torch.empty((n, count), dtype=torch.uint8, device="cuda")
    scales = torch.empty((n, count // 128), dtype=torch.float32, device="cuda")
    y = torch.empty_like(dx)
    assert B.lib().rlx_quantize_fp8(dx.data_ptr(), B.RLX_F32, n, count, count, codes.data_ptr(),
                                    scales.data_ptr(), stream()) == B.RLX_OK
    assert B.lib().rlx_dequantize_fp8(codes.data_ptr(), scales.data_ptr(), n, count, count,
                                      y.data_ptr(), B.RLX_F32, stream()) == B.RLX_OK
    torch.cuda.synchronize()
    oc, os_ = oracle.quantize(x)
    assert_same(to_host(codes), oc, "lp-allreduce quantize codes")
    assert_same(to_host(scales), os_, "lp-allreduce quantize scales")
    assert_same(to_host(y), oracle.dequantize(oc, os_), "lp-allreduce dequantize")


@pytest.mark.parametrize("wire", [FP8, NAT])
def test_workload4_chunked_whole(lp_allreduce, wire):
    """The benchmark step's reduce-scatter, all-gather and alltoall on
    workload 4 (m = 2 Mi): whole outputs; on the FP8 wire reduce-scatter
    then all-gather is the FP8 DDA-tree, bit for bit."""
    x, dx = lp_allreduce
    ag, _ = _check_chunked_whole(x, dx, B.RLX_F32, wire, "lp-allreduce")
    if wire == FP8:
        tree = _allreduce("tree", dx, x.shape[1], FP8, B.RLX_F32)
        assert torch.equal(ag.view(torch.int32), tree.view(torch.int32))


def test_workload4_fp8_error_bound(lp_allreduce):
    """The whole FP8 DDA-flat result lies within the e4m3 error bound of the
    exact (fp64) sum: |w(x) - x| <= 2^-4 |x| + 2^-10 s per element, plus the
    fp32 rounding of the N-term sum, (N-1) u sum |w(x)|."""
    x, dx = lp_allreduce
    n, count = x.shape
    flat = _allreduce("flat", dx, count, FP8, B.RLX_F32)
    blocks = dx.view(n, -1, 128)
    s = (blocks.abs().amax(-1, keepdim=True).double() / 448.0).float().double()
    # e4m3 rounding of fl32(x/s), plus the roundings of the quotient and of
    # the dequantising product (a few units of 2^-24 |x|)
    bound_terms = blocks.abs().double() * (2.0 ** -4 + 2.0 ** -21) + s * 2.0 ** -10 * (1 + 2.0 ** -20)
    bound = bound_terms.sum(0).view(-1)
    bound += (n - 1) * 2.0 ** -24 * (dx.abs().double().sum(0) * (1 + 2.0 ** -3))
    err = (flat[0].double() - dx.double().sum(0)).abs()
    assert bool((err <= bound).all())


# ---------------------------------------------------------------- workload 5

@pytest.fixture(scope="module")
def lp_collectives():
    x = synth.rank_buffers(5)
    return x, to_dev(x)


@pytest.mark.parametrize("wire", [FP8, NAT])
def test_workload5_lp_collectives_whole(lp_collectives, wire):
    """N=8, fp32 [67,108,864] Student-t(3): reduce-scatter (8 Mi per rank),
    all-gather of its result and alltoall, every element against the oracle;
    native alltoall undoes itself; FP8 RS + AG == DDA-tree."""
    x, dx = lp_collectives
    n, count = x.shape
    m = count // n
    ag, a2a = _check_chunked_whole(x, dx, B.RLX_F32, wire, "lp-collectives")
    if wire == NAT:
        back = torch.empty_like(dx)
        assert B.lib().rlx_alltoall(a2a.data_ptr(), count, back.data_ptr(), count, m, n,
                                    B.RLX_F32, NAT, stream()) == B.RLX_OK
        torch.cuda.synchronize()
        assert torch.equal(back.view(torch.int32), dx.view(torch.int32))
    else:
        del a2a
        tree = _allreduce("tree", dx, count, FP8, B.RLX_F32)
        assert torch.equal(ag.view(torch.int32), tree.view(torch.int32))
