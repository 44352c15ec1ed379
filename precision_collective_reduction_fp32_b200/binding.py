"""ctypes binding of librlx.so: one Python function per C entry point, same
names, same arguments (device pointers as ints, sizes, enums, stream handle).

This module only marshals arguments.  Every computation happens in the CUDA
kernels behind the C ABI; if librlx.so is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librlx.so")

# enums of include/rlx.h
RLX_OK, RLX_ERR_INVALID_ARG, RLX_ERR_ALIGNMENT, RLX_ERR_UNSUPPORTED = 0, 1, 2, 3
RLX_ERR_WORKSPACE, RLX_ERR_CUDA, RLX_ERR_TIMEOUT = 4, 5, 6
RLX_F32, RLX_BF16 = 0, 1
RLX_WIRE_NATIVE, RLX_WIRE_FP8_E4M3 = 0, 1
RLX_SUM = 0
RLX_COLL_ALLREDUCE_FLAT, RLX_COLL_ALLREDUCE_TREE, RLX_COLL_REDUCE_SCATTER = 0, 1, 2
RLX_COLL_ALL_GATHER, RLX_COLL_ALLTOALL, RLX_COLL_ALLREDUCE_TREE_FUSED = 3, 4, 5
RLX_TREE_SYNC_BYTES = 256
RLX_DEFAULT_WAIT_NS = 1_000_000_000
RLX_BLOCK = 128
RLX_MAX_RANKS = 16

# every symbol include/rlx.h declares
EXPORTS = ("rlx_quantize_fp8", "rlx_dequantize_fp8", "rlx_allreduce_flat", "rlx_allreduce_tree",
           "rlx_reduce_scatter", "rlx_all_gather", "rlx_alltoall", "rlx_workspace_bytes",
           "rlx_status_string", "rlx_last_cuda_error", "rlx_allreduce_tree_noalloc",
           "rlx_allreduce_tree_fused")
RLX_NOALLOC_MAX_COUNT = 16777216


class RlxError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = "%s: %s" % (where, status_string(status))
        if status == RLX_ERR_CUDA:
            msg += " (cudaError %d)" % lib().rlx_last_cuda_error()
        super().__init__(msg)


_lib = None


def lib() -> ctypes.CDLL:
    """Load librlx.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("librlx.so is not built; run "
                               "`python -m precision_collective_reduction_fp32_b200.build`")
        _lib = load(LIB_PATH)
    return _lib


def load(path: str) -> ctypes.CDLL:
    """A new handle on the build at `path` with every entry point's
    signature set (lib() uses it for the product build; bench.py's ablation
    mode for profiling builds of the same sources)."""
    L = ctypes.CDLL(path)
    P, S, I = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    sig = {
        "rlx_quantize_fp8": [P, I, S, S, S, P, P, P],
        "rlx_dequantize_fp8": [P, P, S, S, S, P, I, P],
        "rlx_allreduce_flat": [P, P, S, S, I, I, I, I, P],
        "rlx_allreduce_tree": [P, P, S, S, I, I, I, I, P, S, P],
        "rlx_allreduce_tree_noalloc": [P, P, S, S, I, I, I, I, P],
        "rlx_allreduce_tree_fused": [P, P, S, S, I, I, I, I, P, S, P, ctypes.c_uint64, P],
        "rlx_reduce_scatter": [P, S, P, S, S, I, I, I, I, P],
        "rlx_all_gather": [P, S, P, S, S, I, I, I, P],
        "rlx_alltoall": [P, S, P, S, S, I, I, I, P],
        "rlx_workspace_bytes": [I, S, I, I, I],
        "rlx_status_string": [I],
        "rlx_last_cuda_error": [],
    }
    for name, args in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = I
    L.rlx_workspace_bytes.restype = S
    L.rlx_status_string.restype = ctypes.c_char_p
    return L


def _call(name: str, *args) -> None:
    st = getattr(lib(), name)(*args)
    if st != RLX_OK:
        raise RlxError(st, name)


def status_string(status: int) -> str:
    return lib().rlx_status_string(status).decode()


def rlx_status_string(status: int) -> str:
    return status_string(status)


def rlx_last_cuda_error() -> int:
    return lib().rlx_last_cuda_error()


def rlx_workspace_bytes(coll: int, count: int, nranks: int, dtype: int, wire: int) -> int:
    return lib().rlx_workspace_bytes(coll, count, nranks, dtype, wire)


def rlx_quantize_fp8(x, dtype, rows, n, stride, codes, scales, stream=None) -> None:
    _call("rlx_quantize_fp8", x, dtype, rows, n, stride, codes, scales, stream)


def rlx_dequantize_fp8(codes, scales, rows, n, stride, y, dtype, stream=None) -> None:
    _call("rlx_dequantize_fp8", codes, scales, rows, n, stride, y, dtype, stream)


def rlx_allreduce_flat(send, recv, count, stride, nranks, dtype, wire, op=RLX_SUM,
                       stream=None) -> None:
    _call("rlx_allreduce_flat", send, recv, count, stride, nranks, dtype, wire, op, stream)


def rlx_allreduce_tree(send, recv, count, stride, nranks, dtype, wire, op=RLX_SUM,
                       workspace=None, workspace_bytes=0, stream=None) -> None:
    _call("rlx_allreduce_tree", send, recv, count, stride, nranks, dtype, wire, op, workspace,
          workspace_bytes, stream)


def rlx_allreduce_tree_noalloc(send, recv, count, stride, nranks, dtype, wire, op=RLX_SUM,
                               stream=None) -> None:
    """DDA-tree allreduce whose FP8 payload sits in the library's fixed
    device array (no workspace argument; count <= RLX_NOALLOC_MAX_COUNT on
    the FP8 wire).  For callers that cannot allocate device memory."""
    _call("rlx_allreduce_tree_noalloc", send, recv, count, stride, nranks, dtype, wire, op, stream)


def rlx_allreduce_tree_fused(send, recv, count, stride, nranks, dtype, wire, op=RLX_SUM,
                             workspace=None, workspace_bytes=0, status=None, wait_limit_ns=0,
                             stream=None) -> None:
    """DDA-tree allreduce in one launch with bounded chunk-ready waits; the
    device int at `status` (if given) receives RLX_OK or RLX_ERR_TIMEOUT."""
    _call("rlx_allreduce_tree_fused", send, recv, count, stride, nranks, dtype, wire, op,
          workspace, workspace_bytes, status, wait_limit_ns, stream)


def rlx_reduce_scatter(send, send_stride, recv, recv_stride, m, nranks, dtype, wire,
                       op=RLX_SUM, stream=None) -> None:
    _call("rlx_reduce_scatter", send, send_stride, recv, recv_stride, m, nranks, dtype, wire,
          op, stream)


def rlx_all_gather(send, send_stride, recv, recv_stride, m, nranks, dtype, wire,
                   stream=None) -> None:
    _call("rlx_all_gather", send, send_stride, recv, recv_stride, m, nranks, dtype, wire, stream)


def rlx_alltoall(send, send_stride, recv, recv_stride, m, nranks, dtype, wire,
                 stream=None) -> None:
    _call("rlx_alltoall", send, send_stride, recv, recv_stride, m, nranks, dtype, wire, stream)
