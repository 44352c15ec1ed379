"""GPU parity at the benchmark sizes, in the layout the benchmark uses.

The five workloads (see precision_collective_reduction_fp32_b200.synth) run
through the C ABI on contiguous [N][count] rank rows.  The oracle cannot
redo 2 GiB at these sizes in a test, so each check is one of:
  * sampled outputs: 128-blocks picked at random (plus first, last, chunk
    edges) are cut out of the inputs, the oracle computes them exactly as it
    would in place (blocks never straddle a chunk, so the arithmetic is the
    same), and the GPU values must match bit for bit;
  * properties that hold at any size, checked on the whole output on the GPU:
    every rank's allreduce result is identical, DDA-tree == DDA-flat on the
    native wire, reduce-scatter then all-gather == DDA-tree on the FP8 wire,
    alltoall is the chunk transpose and undoes itself, and the FP8 results
    stay within the e4m3 error bound of the exact (fp64) sum.
Bar: bit-exact for every sampled value and every property.
"""
import numpy as np
import pytest
import torch

import oracle
import refpipe
from gpuutil import stream, to_dev, to_host
from precision_collective_reduction_fp32_b200 import binding as B
from precision_collective_reduction_fp32_b200 import build as rlx_build
from precision_collective_reduction_fp32_b200 import synth

pytestmark = pytest.mark.gpu

NAT, FP8 = B.RLX_WIRE_NATIVE, B.RLX_WIRE_FP8_E4M3
ORC = {NAT: oracle.NATIVE, FP8: oracle.FP8}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    rlx_build.build()
    oracle.build()


def _sample_blocks(count, nblocks=192, extra=(), seed=0):
    nb = (count + 127) // 128
    rng = np.random.default_rng(seed)
    pick = set(rng.integers(0, nb, size=min(nblocks, nb)).tolist())
    pick |= {0, nb - 1} | {b for b in extra if 0 <= b < nb}
    return sorted(pick)


def _cols(blocks, count, base=0):
    idx = [np.arange(base + b * 128, base + min((b + 1) * 128, count)) for b in blocks]
    return np.concatenate(idx)


def _same(a, b):
    return refpipe.same_bits(a, b)


def _cols_of(t, idx):
    """Columns idx of every row of a device tensor, copied to the host."""
    return to_host(t[:, torch.from_numpy(np.asarray(idx, dtype=np.int64)).cuda()])


def _allreduce(algo, dx, count, wire, dcode):
    n = dx.shape[0]
    out = torch.empty_like(dx)
    if algo == "flat":
        B.rlx_allreduce_flat(dx.data_ptr(), out.data_ptr(), count, count, n, dcode, wire,
                             B.RLX_SUM, stream())
    else:
        need = B.rlx_workspace_bytes(B.RLX_COLL_ALLREDUCE_TREE, count, n, dcode, wire)
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
        B.rlx_allreduce_tree(dx.data_ptr(), out.data_ptr(), count, count, n, dcode, wire,
                             B.RLX_SUM, ws.data_ptr(), need, stream())
    torch.cuda.synchronize()
    return out


def _rows_identical(out):
    flat = out.view(out.shape[0], -1)
    return all(torch.equal(flat[0].view(torch.int16 if flat.dtype == torch.bfloat16 else torch.int32),
                           flat[r].view(torch.int16 if flat.dtype == torch.bfloat16 else torch.int32))
               for r in range(1, flat.shape[0]))


def _check_allreduce_sampled(x, out, algo, wire, count, chunk_edges=()):
    blocks = _sample_blocks(count, extra=chunk_edges)
    idx = _cols(blocks, count)
    xs = np.ascontiguousarray(x[:, idx])
    fn = oracle.allreduce_flat if algo == "flat" else oracle.allreduce_tree
    ref = fn(xs, wire=ORC[wire])
    got = _cols_of(out, idx)
    assert _same(got, ref), (algo, wire)


# ---------------------------------------------------------------- workload 1

@pytest.mark.parametrize("algo", ["flat", "tree"])
@pytest.mark.parametrize("wire", [NAT, FP8])
def test_workload1_tiny_full_compare(algo, wire):
    """N=8, fp32 [10,20]: the whole output against the oracle."""
    x = synth.rank_buffers(1)
    out = _allreduce(algo, to_dev(x), 200, wire, B.RLX_F32)
    fn = oracle.allreduce_flat if algo == "flat" else oracle.allreduce_tree
    assert _same(to_host(out), fn(x, wire=ORC[wire]))


# ---------------------------------------------------------------- workload 2

@pytest.mark.parametrize("wire", [NAT, FP8])
def test_workload2_decode_full_compare(wire):
    """N=8, bf16 [32, 8192]: DDA-flat, fp32 accumulation, bf16 out; whole output."""
    x = synth.rank_buffers(2)
    out = _allreduce("flat", to_dev(x), x.shape[1], wire, B.RLX_BF16)
    assert _same(to_host(out), oracle.allreduce_flat(x, wire=ORC[wire]))


# ---------------------------------------------------------------- workload 3

def test_workload3_prefill_tree():
    """N=8, bf16 [4096, 8192] (64 MiB/rank): DDA-tree native; sampled blocks
    (incl. chunk edges) against the oracle; tree == flat and all rows equal
    on the whole output."""
    x = synth.rank_buffers(3)
    count = x.shape[1]
    dx = to_dev(x)
    tree = _allreduce("tree", dx, count, NAT, B.RLX_BF16)
    C = oracle.tree_chunk(count, 8)
    edges = [c * C // 128 + d for c in range(1, 8) for d in (-1, 0)]
    _check_allreduce_sampled(x, tree, "tree", NAT, count, edges)
    flat = _allreduce("flat", dx, count, NAT, B.RLX_BF16)
    assert torch.equal(tree.view(torch.int16), flat.view(torch.int16))
    assert _rows_identical(tree)
    for wire in (FP8,):
        t8 = _allreduce("tree", dx, count, wire, B.RLX_BF16)
        _check_allreduce_sampled(x, t8, "tree", wire, count, edges)
        assert _rows_identical(t8)
        del t8
        f8 = _allreduce("flat", dx, count, wire, B.RLX_BF16)
        _check_allreduce_sampled(x, f8, "flat", wire, count, edges)
        assert _rows_identical(f8)


# ---------------------------------------------------------------- workload 4

def test_workload4_lp_allreduce():
    """N=8, fp32 [16,777,216] with 1% x100 outliers: FP8 DDA-tree (fused
    dequantise-sum-requantise) and FP8 DDA-flat; sampled blocks against the
    oracle, rows identical, reduce-scatter + all-gather == tree, and the
    whole result within the e4m3 bound of the exact sum."""
    x = synth.rank_buffers(4)
    n, count = x.shape
    m = count // n
    dx = to_dev(x)
    C = oracle.tree_chunk(count, n)
    edges = [c * C // 128 + d for c in range(1, n) for d in (-1, 0)]
    tree = _allreduce("tree", dx, count, FP8, B.RLX_F32)
    flat = _allreduce("flat", dx, count, FP8, B.RLX_F32)
    _check_allreduce_sampled(x, tree, "tree", FP8, count, edges)
    _check_allreduce_sampled(x, flat, "flat", FP8, count, edges)
    assert _rows_identical(tree) and _rows_identical(flat)
    # reduce-scatter then all-gather (FP8) is the FP8 tree, bit for bit
    rs = torch.empty((n, m), dtype=torch.float32, device="cuda")
    ag = torch.empty_like(dx)
    B.rlx_reduce_scatter(dx.data_ptr(), count, rs.data_ptr(), m, m, n, B.RLX_F32, FP8, B.RLX_SUM,
                         stream())
    B.rlx_all_gather(rs.data_ptr(), m, ag.data_ptr(), count, m, n, B.RLX_F32, FP8, stream())
    torch.cuda.synchronize()
    assert torch.equal(ag.view(torch.int32), tree.view(torch.int32))
    # error bound of the whole FP8-flat result against the exact sum:
    # |w(x) - x| <= 2^-4 |x| + 2^-10 s per element (e4m3), plus fp32 rounding
    # of the N-term sum, (N-1) u sum|w(x)|.
    xt = torch.from_numpy(x).cuda()
    blocks = xt.view(n, -1, 128)
    s = (blocks.abs().amax(-1, keepdim=True).double() / 448.0).float().double()
    # e4m3 rounding of fl32(x/s), plus the roundings of the quotient and of
    # the dequantising product (a few units of 2^-24 |x|)
    bound_terms = blocks.abs().double() * (2.0 ** -4 + 2.0 ** -21) + s * 2.0 ** -10 * (1 + 2.0 ** -20)
    bound = bound_terms.sum(0).view(-1)
    bound += (n - 1) * 2.0 ** -24 * (xt.abs().double().sum(0) * (1 + 2.0 ** -3))
    err = (flat[0].double() - xt.double().sum(0)).abs()
    assert bool((err <= bound).all())


# ---------------------------------------------------------------- workload 5

@pytest.mark.parametrize("wire", [FP8, NAT])
def test_workload5_lp_collectives(wire):
    """N=8, fp32 [67,108,864] Student-t(3): reduce-scatter, all-gather and
    alltoall; sampled (chunk, block) outputs against the oracle; alltoall is
    the chunk transpose (native) and RS + AG == DDA-tree (FP8)."""
    x = synth.rank_buffers(5)
    n, count = x.shape
    m = count // n
    dx = to_dev(x)
    rs = torch.empty((n, m), dtype=torch.float32, device="cuda")
    ag = torch.empty_like(dx)
    a2a = torch.empty_like(dx)
    B.rlx_reduce_scatter(dx.data_ptr(), count, rs.data_ptr(), m, m, n, B.RLX_F32, wire, B.RLX_SUM,
                         stream())
    B.rlx_all_gather(rs.data_ptr(), m, ag.data_ptr(), count, m, n, B.RLX_F32, wire, stream())
    B.rlx_alltoall(dx.data_ptr(), count, a2a.data_ptr(), count, m, n, B.RLX_F32, wire, stream())
    torch.cuda.synchronize()
    blocks = _sample_blocks(m, nblocks=48, seed=5)
    idx = _cols(blocks, m)
    L = idx.size
    # reduce-scatter: chunk r of every rank, sampled columns
    xs = np.zeros((n, n * L), dtype=np.float32)
    for r in range(n):
        xs[:, r * L:(r + 1) * L] = x[:, r * m + idx]
    ref_rs = oracle.reduce_scatter(xs, L, wire=ORC[wire])
    got_rs = _cols_of(rs, idx)
    assert _same(got_rs, ref_rs)
    # all-gather of the reduce-scatter output, sampled columns
    ref_ag = oracle.all_gather(np.ascontiguousarray(got_rs), L, wire=ORC[wire])
    for s in range(n):
        assert _same(_cols_of(ag, s * m + idx), ref_ag[:, s * L:(s + 1) * L])
    # alltoall, sampled columns of every (s, r) chunk
    ref_a2a = oracle.alltoall(xs, L, wire=ORC[wire])
    for s in range(n):
        assert _same(_cols_of(a2a, s * m + idx), ref_a2a[:, s * L:(s + 1) * L])
    if wire == NAT:
        t = dx.view(n, n, m).transpose(0, 1).reshape(n, count)
        assert torch.equal(a2a.view(torch.int32), t.view(torch.int32))
        back = torch.empty_like(dx)
        B.rlx_alltoall(a2a.data_ptr(), count, back.data_ptr(), count, m, n, B.RLX_F32, NAT, stream())
        torch.cuda.synchronize()
        assert torch.equal(back.view(torch.int32), dx.view(torch.int32))
    else:
        tree = _allreduce("tree", dx, count, FP8, B.RLX_F32)
        assert torch.equal(ag.view(torch.int32), tree.view(torch.int32))
