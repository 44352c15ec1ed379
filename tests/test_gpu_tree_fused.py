"""rlx_allreduce_tree_fused: the DDA-tree allreduce in one launch, with
per-chunk ready counts and bounded waits between its reduce-scatter and
all-gather work.

Parity: every allreduce shape of the parity suite (ragged counts, partial
blocks, 2..16 ranks, padded and unaligned strides), both dtypes and both
wires, against the oracle's DDA-tree bit for bit, with guard bands around
every buffer; the status word must read RLX_OK and the workspace's
synchronisation words must be zero again after every call (the contract that
lets the next call reuse the workspace).  The full decode and lp-allreduce
workloads are compared element by element.

Failure detection: a call whose chunk-ready counts can never reach their
targets (the test presets them to INT_MIN, so the ready flag is one nothing
ever sets) must come back
within its short wait limit with RLX_ERR_TIMEOUT in the status word, leave
the synchronisation words zero, and leave the context usable: the next call
on the same workspace is correct.
"""
import time

import pytest
import torch

import oracle
import refpipe
from gpuutil import Guarded, dcode, guarded_from, stream, to_dev, to_host
from precision_collective_reduction_fp32_b200 import binding as B
from precision_collective_reduction_fp32_b200 import build as rlx_build
from precision_collective_reduction_fp32_b200 import synth

pytestmark = pytest.mark.gpu

NAT, FP8 = B.RLX_WIRE_NATIVE, B.RLX_WIRE_FP8_E4M3
ORC = {NAT: oracle.NATIVE, FP8: oracle.FP8}

CASES = [(n, c) for n in (2, 3, 8) for c in (1, 7, 127, 128, 129, 1000, 3 * 128 * 8 + 5)] + \
        [(4, 4096), (5, 1003), (16, 2000), (8, 65536 + 4), (8, 128 * 1024 + 3)]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    rlx_build.build()
    oracle.build()
    B.lib()


class Fused:
    """A guarded, zeroed workspace and a status word, reused across calls."""

    def __init__(self, count, n, d, wire):
        self.need = B.rlx_workspace_bytes(B.RLX_COLL_ALLREDUCE_TREE_FUSED, count, n, d, wire)
        self.ws = Guarded((max(self.need, 16),), torch.uint8, fill=torch.zeros(max(self.need, 16),
                                                                                 dtype=torch.uint8))
        self.status = torch.full((1,), -1, dtype=torch.int32, device="cuda")

    def call(self, send, recv, count, stride, n, d, wire, limit_ns=0):
        return B.lib().rlx_allreduce_tree_fused(send, recv, count, stride, n, d, wire, B.RLX_SUM,
                                                self.ws.ptr() if self.need else None, self.need,
                                                self.status.data_ptr(), limit_ns, stream())

    def sync_words(self):
        return self.ws.t[:B.RLX_TREE_SYNC_BYTES].view(torch.int32).cpu().numpy()


def _run(x, count, stride, wire, fz=None, offset=0, inplace=False):
    n = x.shape[0]
    d = dcode(x)
    gs = guarded_from(x, offset)
    gr = gs if inplace else Guarded(x.shape, gs.t.dtype, offset,
                                    fill=torch.zeros(x.shape, dtype=gs.t.dtype))
    fz = fz or Fused(count, n, d, wire)
    assert fz.call(gs.ptr(), gr.ptr(), count, stride, n, d, wire) == B.RLX_OK
    torch.cuda.synchronize()
    assert int(fz.status.item()) == B.RLX_OK
    assert gs.guards_intact() and gr.guards_intact() and fz.ws.guards_intact()
    if fz.need:
        assert not fz.sync_words().any(), "synchronisation words not cleared"
    return to_host(gr.t), fz


@pytest.mark.parametrize("wire", [NAT, FP8])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("nranks,count", CASES)
def test_fused_tree_matches_oracle(wire, dtype, nranks, count):
    fz = None   # one workspace for all four layouts: each call must leave it reusable
    for stride, off in ((count, 0), (count + 3, 0), ((count + 7) // 8 * 8, 0), (count, 1)):
        x = synth.rank_buffers(4, count=count, nranks=nranks, stride=stride, dtype=dtype)
        got, fz = _run(x, count, stride, wire, fz, off)
        ref = oracle.allreduce_tree(x, wire=ORC[wire], count=count)
        assert refpipe.same_bits(got[:, :count], ref[:, :count]), (stride, off)
        assert not got[:, count:].any()


@pytest.mark.parametrize("wire", [NAT, FP8])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_fused_tree_inplace_and_reuse(wire, dtype):
    """In place, then three more calls on one workspace with new inputs."""
    n, count = 8, 3000
    fz = Fused(count, n, B.RLX_F32 if dtype == "f32" else B.RLX_BF16, wire)
    for k, wl in enumerate((4, 5, 1, 2)):
        x = synth.rank_buffers(wl, count=count, nranks=n, dtype=dtype)
        got, _ = _run(x, count, count, wire, fz, inplace=(k == 0))
        assert refpipe.same_bits(got, oracle.allreduce_tree(x, wire=ORC[wire])), k


@pytest.mark.parametrize("wire", [NAT, FP8])
def test_fused_tree_decode_workload(wire):
    """N=8 bf16 [32, 8192] (the decode message): whole output."""
    x = synth.rank_buffers(2)
    got, _ = _run(x, x.shape[1], x.shape[1], wire)
    assert refpipe.same_bits(got, oracle.allreduce_tree(x, wire=ORC[wire]))


def test_fused_tree_lp_allreduce_workload():
    """N=8 fp32 [16,777,216] with outliers, FP8 wire: whole output."""
    x = synth.rank_buffers(4)
    n, count = x.shape
    dx = to_dev(x)
    out = torch.empty_like(dx)
    fz = Fused(count, n, B.RLX_F32, FP8)
    assert fz.call(dx.data_ptr(), out.data_ptr(), count, count, n, B.RLX_F32, FP8) == B.RLX_OK
    torch.cuda.synchronize()
    assert int(fz.status.item()) == B.RLX_OK and not fz.sync_words().any()
    assert refpipe.same_bits(to_host(out), oracle.allreduce_tree(x, wire=oracle.FP8))


@pytest.mark.parametrize("wire", [NAT, FP8])
@pytest.mark.parametrize("count", [1000, 262_144])
def test_fused_tree_wait_runs_out(wire, count):
    """Ready counts that can never reach their targets: the call ends within
    its 2 ms wait limit with RLX_ERR_TIMEOUT, clears the synchronisation
    words, and the context and the workspace stay usable."""
    n = 8
    x = synth.rank_buffers(4, count=count, nranks=n)
    dx = to_dev(x)
    out = torch.zeros_like(dx)
    fz = Fused(count, n, B.RLX_F32, wire)
    # word 4 + c counts chunk c's finished reduce-scatter work, compared with
    # its target as a signed number; from INT_MIN the kernel's additions can
    # never reach the target (before or after they land)
    words = fz.ws.t[:B.RLX_TREE_SYNC_BYTES].view(torch.int32)
    words[4:4 + n] = -2 ** 31
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    assert fz.call(dx.data_ptr(), out.data_ptr(), count, count, n, B.RLX_F32, wire,
                   limit_ns=2_000_000) == B.RLX_OK
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(fz.status.item()) == B.RLX_ERR_TIMEOUT
    assert elapsed < 5.0, elapsed
    assert not fz.sync_words().any(), "synchronisation words not cleared after the timeout"
    assert fz.ws.guards_intact()
    # the same workspace works again, and the result is right
    fz.status.fill_(-1)
    assert fz.call(dx.data_ptr(), out.data_ptr(), count, count, n, B.RLX_F32, wire) == B.RLX_OK
    torch.cuda.synchronize()
    assert int(fz.status.item()) == B.RLX_OK
    assert refpipe.same_bits(to_host(out), oracle.allreduce_tree(x, wire=ORC[wire]))


def test_fused_tree_one_rank_and_empty_write_status():
    x = synth.rank_buffers(4, count=500, nranks=1)
    got, _ = _run(x, 500, 500, FP8)
    assert refpipe.same_bits(got, x)
    fz = Fused(0, 8, B.RLX_F32, FP8)
    assert fz.call(0, 0, 0, 0, 8, B.RLX_F32, FP8) == B.RLX_OK
    torch.cuda.synchronize()
    assert int(fz.status.item()) == B.RLX_OK


def test_fused_tree_python_helper():
    """rlx.allreduce(algo="tree_fused") allocates a zeroed workspace itself."""
    import precision_collective_reduction_fp32_b200 as rlx
    x = synth.rank_buffers(3, count=40_000, nranks=4)
    dx = to_dev(x)
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for wire, ow in (("native", oracle.NATIVE), ("fp8", oracle.FP8)):
        y = rlx.allreduce(dx, algo="tree_fused", wire=wire, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == B.RLX_OK
        assert refpipe.same_bits(to_host(y), oracle.allreduce_tree(x, wire=ow))
