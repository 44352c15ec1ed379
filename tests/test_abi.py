"""The C ABI boundary without a GPU: librlx.so loads, exports exactly what
include/rlx.h declares, and rejects bad arguments before any CUDA call.

The pointers below are plain integers that are never dereferenced: every
call here fails validation (or has nothing to do), so nothing is launched.
"""
import os
import re
import subprocess

import pytest

from precision_collective_reduction_fp32_b200 import binding as B
from precision_collective_reduction_fp32_b200 import build as rlx_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
A = 0x7f0000000000   # a 256-byte aligned fake device address
Z = 1 << 30          # distance between fake buffers (no overlap)


@pytest.fixture(scope="module")
def L():
    rlx_build.build()
    return B.lib()


def _declared():
    text = open(os.path.join(ROOT, "include", "rlx.h")).read()
    return sorted(set(re.findall(r"RLX_API\s+[\w\s\*]*?\b(rlx_\w+)\s*\(", text)))


def test_exports_match_header(L):
    declared = _declared()
    assert declared == sorted(B.EXPORTS)
    out = subprocess.check_output(["nm", "-D", "--defined-only", B.LIB_PATH], text=True)
    exported = sorted(l.split()[-1] for l in out.splitlines() if l.split()[-1].startswith("rlx_"))
    assert exported == declared
    for name in declared:
        assert hasattr(L, name)


def test_status_strings(L):
    for s in range(7):
        assert B.rlx_status_string(s) not in ("", "unknown status")
    assert B.rlx_status_string(99) == "unknown status"


def test_workspace_bytes(L):
    f = B.rlx_workspace_bytes
    assert f(B.RLX_COLL_ALLREDUCE_TREE, 1000, 8, B.RLX_F32, B.RLX_WIRE_FP8_E4M3) == 1280
    assert f(B.RLX_COLL_ALLREDUCE_TREE, 16_777_216, 8, B.RLX_F32, B.RLX_WIRE_FP8_E4M3) == \
        16_777_216 + 16_777_216 // 128 * 4
    assert f(B.RLX_COLL_ALLREDUCE_TREE, 1000, 8, B.RLX_F32, B.RLX_WIRE_NATIVE) == 0
    assert f(B.RLX_COLL_ALLREDUCE_TREE, 1000, 1, B.RLX_F32, B.RLX_WIRE_FP8_E4M3) == 0
    assert f(B.RLX_COLL_ALLREDUCE_FLAT, 1000, 8, B.RLX_F32, B.RLX_WIRE_FP8_E4M3) == 0
    # the one-launch tree: sync words, then the FP8 payload
    assert f(B.RLX_COLL_ALLREDUCE_TREE_FUSED, 1000, 8, B.RLX_F32, B.RLX_WIRE_NATIVE) == 256
    assert f(B.RLX_COLL_ALLREDUCE_TREE_FUSED, 1000, 8, B.RLX_F32, B.RLX_WIRE_FP8_E4M3) == 256 + 1280
    assert f(B.RLX_COLL_ALLREDUCE_TREE_FUSED, 1000, 1, B.RLX_F32, B.RLX_WIRE_FP8_E4M3) == 0


def _st(name, *args):
    return getattr(B.lib(), name)(*args)


F32, BF, NAT, FP8, SUM = B.RLX_F32, B.RLX_BF16, B.RLX_WIRE_NATIVE, B.RLX_WIRE_FP8_E4M3, B.RLX_SUM


def test_allreduce_validation(L):
    for name in ("rlx_allreduce_flat", "rlx_allreduce_tree"):
        extra = (None, 0, None) if name.endswith("tree") else (None,)
        ok = (A, A + Z, 100, 100, 8, F32, NAT, SUM)
        call = lambda *a: _st(name, *a, *extra)
        assert call(A, A + Z, 0, 100, 8, F32, NAT, SUM) == B.RLX_OK          # empty: no launch
        assert call(None, A + Z, 100, 100, 8, F32, NAT, SUM) == B.RLX_ERR_INVALID_ARG
        assert call(A, None, 100, 100, 8, F32, NAT, SUM) == B.RLX_ERR_INVALID_ARG
        assert call(A, A + Z, 100, 99, 8, F32, NAT, SUM) == B.RLX_ERR_INVALID_ARG   # stride < count
        assert call(A, A + Z, 100, 100, 0, F32, NAT, SUM) == B.RLX_ERR_INVALID_ARG
        assert call(A, A + Z, 100, 100, 17, F32, NAT, SUM) == B.RLX_ERR_INVALID_ARG
        assert call(A, A + Z, 100, 100, 8, 7, NAT, SUM) == B.RLX_ERR_INVALID_ARG
        assert call(A, A + Z, 100, 100, 8, F32, 5, SUM) == B.RLX_ERR_INVALID_ARG
        assert call(A, A + Z, 100, 100, 8, F32, NAT, 1) == B.RLX_ERR_UNSUPPORTED
        assert call(A + 2, A + Z, 100, 100, 8, F32, NAT, SUM) == B.RLX_ERR_ALIGNMENT
        assert call(A, A + Z + 1, 100, 100, 8, BF, NAT, SUM) == B.RLX_ERR_ALIGNMENT
        assert call(A, A + 400, 100, 100, 8, F32, NAT, SUM) == B.RLX_ERR_INVALID_ARG  # partial overlap
        assert call(A, A + Z, 2 ** 62, 2 ** 62, 8, F32, NAT, SUM) == B.RLX_ERR_INVALID_ARG  # overflow


def test_tree_workspace_validation(L):
    need = B.rlx_workspace_bytes(B.RLX_COLL_ALLREDUCE_TREE, 1000, 8, F32, FP8)
    args = (A, A + Z, 1000, 1000, 8, F32, FP8, SUM)
    assert _st("rlx_allreduce_tree", *args, None, 0, None) == B.RLX_ERR_WORKSPACE
    assert _st("rlx_allreduce_tree", *args, A + 2 * Z, need - 1, None) == B.RLX_ERR_WORKSPACE
    assert _st("rlx_allreduce_tree", *args, A + 2 * Z + 8, need, None) == B.RLX_ERR_WORKSPACE
    assert _st("rlx_allreduce_tree", *args, A + 64, need, None) == B.RLX_ERR_WORKSPACE  # overlaps send


def test_chunked_validation(L):
    # reduce-scatter: send [N][>= N*m], recv [N][>= m]
    rs = lambda *a: _st("rlx_reduce_scatter", *a, None)
    assert rs(A, 799, A + Z, 100, 100, 8, F32, NAT, SUM) == B.RLX_ERR_INVALID_ARG
    assert rs(A, 800, A + Z, 99, 100, 8, F32, NAT, SUM) == B.RLX_ERR_INVALID_ARG
    assert rs(A, 800, A + 64, 100, 100, 8, F32, NAT, SUM) == B.RLX_ERR_INVALID_ARG  # overlap
    assert rs(A, 800, A + Z, 100, 0, 8, F32, NAT, SUM) == B.RLX_OK
    assert rs(A, 800, A + Z, 100, 100, 8, F32, NAT, 3) == B.RLX_ERR_UNSUPPORTED
    ag = lambda *a: _st("rlx_all_gather", *a, None)
    assert ag(A, 99, A + Z, 800, 100, 8, F32, NAT) == B.RLX_ERR_INVALID_ARG
    assert ag(A, 100, A + Z, 799, 100, 8, F32, NAT) == B.RLX_ERR_INVALID_ARG
    assert ag(A, 100, A + Z, 800, 0, 8, F32, FP8) == B.RLX_OK
    assert ag(None, 100, A + Z, 800, 100, 8, F32, NAT) == B.RLX_ERR_INVALID_ARG
    a2 = lambda *a: _st("rlx_alltoall", *a, None)
    assert a2(A, 799, A + Z, 800, 100, 8, F32, NAT) == B.RLX_ERR_INVALID_ARG
    assert a2(A, 800, A + Z, 799, 100, 8, F32, NAT) == B.RLX_ERR_INVALID_ARG
    assert a2(A, 800, A + 4, 800, 100, 8, F32, NAT) == B.RLX_ERR_INVALID_ARG
    assert a2(A + 1, 800, A + Z, 800, 100, 8, BF, NAT) == B.RLX_ERR_ALIGNMENT
    assert a2(A, 800, A + Z, 800, 100, 0, F32, NAT) == B.RLX_ERR_INVALID_ARG
    assert a2(A, 2 ** 62, A + Z, 2 ** 62, 2 ** 61, 8, F32, NAT) == B.RLX_ERR_INVALID_ARG


def test_quant_validation(L):
    q = lambda *a: _st("rlx_quantize_fp8", *a, None)
    assert q(A, F32, 2, 100, 99, A + Z, A + 2 * Z) == B.RLX_ERR_INVALID_ARG
    assert q(A, F32, 0, 100, 100, A + Z, A + 2 * Z) == B.RLX_OK
    assert q(None, F32, 2, 100, 100, A + Z, A + 2 * Z) == B.RLX_ERR_INVALID_ARG
    assert q(A + 1, BF, 2, 100, 100, A + Z, A + 2 * Z) == B.RLX_ERR_ALIGNMENT
    assert q(A, F32, 2, 100, 100, A + Z, A + 2 * Z + 2) == B.RLX_ERR_ALIGNMENT
    assert q(A, F32, 2, 100, 100, A + 100, A + 2 * Z) == B.RLX_ERR_INVALID_ARG  # codes overlap x
    d = lambda *a: _st("rlx_dequantize_fp8", *a, None)
    assert d(A, A + Z, 2, 100, 100, A + 2 * Z, 9) == B.RLX_ERR_INVALID_ARG
    assert d(A, A + Z, 2, 100, 100, A + 16, F32) == B.RLX_ERR_INVALID_ARG     # y overlaps codes
    assert d(A, A + Z + 1, 2, 100, 100, A + 2 * Z, F32) == B.RLX_ERR_ALIGNMENT


def test_element_limit(L):
    """2^36 elements per call (all ranks) at most; one more is rejected before
    any CUDA call (the pointers here are never touched)."""
    big = (1 << 36) // 8 + 1
    assert _st("rlx_allreduce_flat", A, A + (1 << 40), big, big, 8, F32, NAT, SUM, None) == \
        B.RLX_ERR_INVALID_ARG
    assert _st("rlx_allreduce_tree", A, A + (1 << 40), big, big, 8, F32, FP8, SUM, None, 0, None) == \
        B.RLX_ERR_INVALID_ARG
    assert _st("rlx_alltoall", A, 8 * big, A + (1 << 42), 8 * big, big, 8, F32, NAT, None) == \
        B.RLX_ERR_INVALID_ARG
    assert _st("rlx_quantize_fp8", A, F32, 8, big, big, A + (1 << 40), A + (1 << 41), None) == \
        B.RLX_ERR_INVALID_ARG


def test_no_cuda_error_recorded(L):
    """None of the rejected calls above reached CUDA."""
    assert B.rlx_last_cuda_error() == 0


def test_binding_raises_without_gpu_work(L):
    with pytest.raises(B.RlxError) as e:
        B.rlx_allreduce_flat(A, A + Z, 100, 99, 8, F32, NAT)
    assert e.value.status == B.RLX_ERR_INVALID_ARG


def test_build_flags_keep_ieee_rounding():
    """Parity with the oracle depends on these: no multiply-add contraction,
    correctly rounded division and square root, subnormals kept, and code
    for sm_100a only."""
    from precision_collective_reduction_fp32_b200 import build
    f = build.FLAGS
    for flag in ("-fmad=false", "-prec-div=true", "-prec-sqrt=true", "-ftz=false"):
        assert flag in f
    assert "arch=compute_100a,code=sm_100a" in f
    assert not any(x.startswith("--use_fast_math") or x == "-use_fast_math" for x in f)


def test_fused_tree_rejects_before_launch(L):
    """Bad arguments and bad workspaces of rlx_allreduce_tree_fused come back
    as status codes before anything is launched."""
    F, FP8, NAT = B.RLX_F32, B.RLX_WIRE_FP8_E4M3, B.RLX_WIRE_NATIVE
    need = B.rlx_workspace_bytes(B.RLX_COLL_ALLREDUCE_TREE_FUSED, 1000, 8, F, FP8)
    ws, st = A + 4 * Z, A + 5 * Z
    call = lambda *a: _st("rlx_allreduce_tree_fused", *a)
    assert call(A, A + Z, 1000, 1000, 8, F, FP8, B.RLX_SUM, None, 0, st, 0, None) == B.RLX_ERR_WORKSPACE
    assert call(A, A + Z, 1000, 1000, 8, F, FP8, B.RLX_SUM, ws, need - 1, st, 0, None) == B.RLX_ERR_WORKSPACE
    assert call(A, A + Z, 1000, 1000, 8, F, NAT, B.RLX_SUM, ws + 8, 256, st, 0, None) == B.RLX_ERR_WORKSPACE
    assert call(A, A + Z, 1000, 1000, 8, F, FP8, B.RLX_SUM, A + 16, need, st, 0, None) == B.RLX_ERR_WORKSPACE
    assert call(A, A + Z, 1000, 1000, 8, F, FP8, B.RLX_SUM, ws, need, st + 2, 0, None) == B.RLX_ERR_ALIGNMENT
    assert call(A, A + Z, 1000, 1000, 8, F, FP8, B.RLX_SUM, ws, need, A + 64, 0, None) == B.RLX_ERR_INVALID_ARG
    assert call(A, A + Z, 1000, 1000, 8, F, FP8, 1, ws, need, st, 0, None) == B.RLX_ERR_UNSUPPORTED
    assert call(A, A + Z, 1000, 999, 8, F, FP8, B.RLX_SUM, ws, need, st, 0, None) == B.RLX_ERR_INVALID_ARG
    assert call(A, A + Z, 1000, 1000, 17, F, FP8, B.RLX_SUM, ws, need, st, 0, None) == B.RLX_ERR_INVALID_ARG
    assert call(None, A + Z, 1000, 1000, 8, F, FP8, B.RLX_SUM, ws, need, st, 0, None) == B.RLX_ERR_INVALID_ARG
