"""rlx_allreduce_tree_noalloc: the DDA-tree allreduce for callers that cannot
allocate device memory (no workspace argument; the FP8 payload sits in a
fixed device array inside the library).

Each case calls the new entry point through the C ABI twice in a row, on two
different inputs, and compares each result with rlx_allreduce_tree given a
workspace allocated here -- bit for bit, the bar of every parity test in
this suite (the arithmetic is the same; only where the payload lives
differs).  The second call also shows that the payload left behind by the
first call does not leak into the next result.  Two FP8 cases are also
compared with the CPU oracle's DDA-tree, again on two calls in a row.
This file is collected last and works on its own in a fresh process (it
builds and loads the library itself).
"""
import numpy as np
import pytest
import torch

import oracle
from precision_collective_reduction_fp32_b200 import binding as B
from precision_collective_reduction_fp32_b200 import build as rlx_build
from precision_collective_reduction_fp32_b200 import synth

pytestmark = pytest.mark.gpu

CASES = [  # (nranks, count, stride, dtype, wire)
    (8, 1000, 1000, torch.float32, B.RLX_WIRE_FP8_E4M3),
    (8, 4096 * 128 + 37, 4096 * 128 + 40, torch.float32, B.RLX_WIRE_FP8_E4M3),
    (3, 20000, 20003, torch.bfloat16, B.RLX_WIRE_FP8_E4M3),
    (8, B.RLX_NOALLOC_MAX_COUNT, B.RLX_NOALLOC_MAX_COUNT, torch.float32, B.RLX_WIRE_FP8_E4M3),
    (8, 5000, 5000, torch.float32, B.RLX_WIRE_NATIVE),
]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    rlx_build.build()
    oracle.build()
    B.lib()


def _dcode(dt):
    return B.RLX_F32 if dt == torch.float32 else B.RLX_BF16


def _bits(t):
    return t.view(torch.int32 if t.dtype == torch.float32 else torch.int16)


def _with_workspace(x, count, stride, wire):
    n = x.shape[0]
    need = B.rlx_workspace_bytes(B.RLX_COLL_ALLREDUCE_TREE, count, n, _dcode(x.dtype), wire)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    out = torch.zeros_like(x)
    B.rlx_allreduce_tree(x.data_ptr(), out.data_ptr(), count, stride, n, _dcode(x.dtype), wire,
                         B.RLX_SUM, ws.data_ptr() if need else None, need, None)
    return out


def _no_alloc(x, count, stride, wire):
    n = x.shape[0]
    out = torch.zeros_like(x)
    B.rlx_allreduce_tree_noalloc(x.data_ptr(), out.data_ptr(), count, stride, n, _dcode(x.dtype),
                                 wire, B.RLX_SUM, None)
    return out


@pytest.mark.parametrize("nranks,count,stride,dtype,wire", CASES)
def test_no_alloc_matches_workspace_version_twice(nranks, count, stride, dtype, wire):
    g = torch.Generator(device="cuda").manual_seed(count + nranks)
    for call in range(2):
        x = (torch.randn((nranks, stride), generator=g, device="cuda") * (1 + 99 * call)).to(dtype)
        ref = _with_workspace(x, count, stride, wire)
        got = _no_alloc(x, count, stride, wire)
        torch.cuda.synchronize()
        assert torch.equal(_bits(got), _bits(ref)), "call %d differs" % call


def test_no_alloc_rejects_counts_above_the_fixed_payload():
    n, count = 2, B.RLX_NOALLOC_MAX_COUNT + 1
    x = torch.zeros((n, count), dtype=torch.float32, device="cuda")
    st = B.lib().rlx_allreduce_tree_noalloc(x.data_ptr(), x.data_ptr(), count, count, n, B.RLX_F32,
                                            B.RLX_WIRE_FP8_E4M3, B.RLX_SUM, None)
    assert st == B.RLX_ERR_WORKSPACE
    # the native wire needs no payload, so it has no such limit
    B.rlx_allreduce_tree_noalloc(x.data_ptr(), x.data_ptr(), count, count, n, B.RLX_F32,
                                 B.RLX_WIRE_NATIVE, B.RLX_SUM, None)
    torch.cuda.synchronize()


@pytest.mark.parametrize("workload,nranks,count", [(4, 8, 300_000 + 77), (3, 5, 100_003)])
def test_no_alloc_matches_oracle_twice(workload, nranks, count):
    """Two calls in a row on two seeded inputs (first the workload's own
    recipe and seeds, then the Student-t recipe of workload 5): every element
    of every rank equals the oracle's FP8 DDA-tree."""
    for call, wl in enumerate((workload, 5)):
        x = synth.rank_buffers(wl, count=count, nranks=nranks,
                               dtype=synth.WORKLOADS[workload].dtype)
        xt = torch.from_numpy(x.view(np.int16) if x.dtype == np.uint16 else x).cuda()
        out = torch.zeros_like(xt)
        d = B.RLX_BF16 if x.dtype == np.uint16 else B.RLX_F32
        B.rlx_allreduce_tree_noalloc(xt.data_ptr(), out.data_ptr(), count, count, nranks, d,
                                     B.RLX_WIRE_FP8_E4M3, B.RLX_SUM, None)
        torch.cuda.synchronize()
        got = out.cpu().numpy().view(x.dtype)
        ref = oracle.allreduce_tree(x, wire=oracle.FP8)
        assert np.array_equal(got.view(np.uint8), ref.view(np.uint8)), "call %d differs" % call
