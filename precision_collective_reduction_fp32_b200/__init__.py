"""B200-native emulated RCCLX collectives.

N simulated ranks are the rows of one CUDA tensor ``[N, ...]`` on one GPU.
The functions below take torch CUDA tensors, pass their device pointers,
strides and the current CUDA stream to librlx.so (include/rlx.h) and return
torch tensors.  PyTorch only allocates memory and supplies the stream; every
step of every collective runs in the library's CUDA kernels.  There is no CPU
path: without librlx.so every call raises.

    import precision_collective_reduction_fp32_b200 as rlx
    x = torch.randn(8, 10, 20, device="cuda")           # rank r = x[r]
    y = rlx.allreduce(x, algo="tree", wire="fp8")        # [8, 10, 20]
"""
from __future__ import annotations

import os

import torch

from . import binding as _b
from .binding import (RLX_BF16, RLX_BLOCK, RLX_COLL_ALL_GATHER, RLX_COLL_ALLREDUCE_FLAT,
                      RLX_COLL_ALLREDUCE_TREE, RLX_COLL_ALLREDUCE_TREE_FUSED, RLX_COLL_ALLTOALL,
                      RLX_COLL_REDUCE_SCATTER, RLX_ERR_TIMEOUT, RLX_F32, RLX_MAX_RANKS, RLX_OK,
                      RLX_SUM, RLX_WIRE_FP8_E4M3, RLX_WIRE_NATIVE, RlxError, rlx_all_gather,
                      rlx_allreduce_flat, rlx_allreduce_tree, rlx_allreduce_tree_fused,
                      rlx_allreduce_tree_noalloc, rlx_alltoall, rlx_dequantize_fp8,
                      rlx_quantize_fp8, rlx_reduce_scatter, rlx_status_string,
                      rlx_workspace_bytes)

__all__ = ["allreduce", "reduce_scatter", "all_gather", "alltoall", "quantize_fp8",
           "dequantize_fp8", "workspace_bytes", "RlxError", "rlx_allreduce_flat",
           "rlx_allreduce_tree", "rlx_allreduce_tree_noalloc", "rlx_allreduce_tree_fused",
           "rlx_reduce_scatter",
           "rlx_all_gather", "rlx_alltoall", "rlx_quantize_fp8", "rlx_dequantize_fp8",
           "rlx_workspace_bytes", "rlx_status_string", "default_wire"]

_WIRES = {"native": RLX_WIRE_NATIVE, "fp8": RLX_WIRE_FP8_E4M3}


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return RLX_F32
    if t.dtype == torch.bfloat16:
        return RLX_BF16
    raise TypeError("rank buffers must be float32 or bfloat16, got %s" % t.dtype)


def _rows(t: torch.Tensor) -> tuple[int, int, int]:
    """(nranks, elements per rank, row stride) of a [N, ...] CUDA tensor whose
    rows are each contiguous."""
    if not t.is_cuda:
        raise ValueError("rank buffers must be CUDA tensors")
    if t.dim() < 1:
        raise ValueError("rank buffers are [N, ...] tensors")
    n = t.shape[0]
    per = t[0].numel() if n else 0
    if t.dim() == 1:
        return n, 1, t.stride(0)
    inner = t[0]
    if not inner.is_contiguous():
        raise ValueError("each rank's row must be contiguous")
    return n, per, t.stride(0)


def _stream():
    return ctypes_stream(torch.cuda.current_stream())


def ctypes_stream(s: torch.cuda.Stream):
    return s.cuda_stream or None


# The pages switch the low-precision collectives on for a whole job with an
# environment variable ("Coletivos de Baixa Precisão", infolabhq pt:
# RCCL_LOW_PRECISION_ENABLE=1) and let users enable them selectively.  Here a
# call with wire=None takes the FP8 wire when RLX_LOW_PRECISION_ENABLE (or
# the pages' RCCL_LOW_PRECISION_ENABLE) is "1", else the native wire; an
# explicit wire= always wins.
LOW_PRECISION_ENV = ("RLX_LOW_PRECISION_ENABLE", "RCCL_LOW_PRECISION_ENABLE")


def default_wire() -> str:
    return "fp8" if any(os.environ.get(v) == "1" for v in LOW_PRECISION_ENV) else "native"


def _wire(w: str | None) -> int:
    if w is None:
        w = default_wire()
    try:
        return _WIRES[w]
    except KeyError:
        raise ValueError("wire must be 'native' or 'fp8'") from None


def workspace_bytes(coll: int, count: int, nranks: int, dtype: torch.dtype,
                    wire: str | None = None) -> int:
    d = RLX_F32 if dtype == torch.float32 else RLX_BF16
    return rlx_workspace_bytes(coll, count, nranks, d, _wire(wire))


def fused_tree_workspace(x: torch.Tensor, wire: str | None = None) -> torch.Tensor:
    """A zeroed workspace for algo="tree_fused" on rank buffers shaped like x
    (reusable by later calls on the same stream: each call leaves its
    synchronisation words zero)."""
    n, count, _ = _rows(x)
    need = rlx_workspace_bytes(RLX_COLL_ALLREDUCE_TREE_FUSED, count, n, _dtype(x), _wire(wire))
    return torch.zeros(max(need, 16), dtype=torch.uint8, device=x.device)


def allreduce(x: torch.Tensor, algo: str = "flat", wire: str | None = None,
              out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
              status: torch.Tensor | None = None, wait_limit_ns: int = 0):
    """SUM allreduce over the ranks (rows) of x.  out may be x (in place).

    algo: "flat" (DDA-flat), "tree" (DDA-tree, two launches) or "tree_fused"
    (DDA-tree in one launch with bounded chunk-ready waits; its workspace
    must start zeroed, see fused_tree_workspace, and `status`, an int32 CUDA
    tensor of one element, receives RLX_OK or RLX_ERR_TIMEOUT)."""
    n, count, stride = _rows(x)
    out = torch.empty_like(x) if out is None else out
    if out.shape != x.shape or out.dtype != x.dtype or _rows(out)[2] != stride:
        raise ValueError("out must match x in shape, dtype and row stride")
    d, w = _dtype(x), _wire(wire)
    if status is not None and algo != "tree_fused":
        raise ValueError("status applies to algo='tree_fused' only")
    if algo == "flat":
        rlx_allreduce_flat(x.data_ptr(), out.data_ptr(), count, stride, n, d, w, RLX_SUM, _stream())
    elif algo == "tree":
        need = rlx_workspace_bytes(RLX_COLL_ALLREDUCE_TREE, count, n, d, w)
        if need and workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
        wp = workspace.data_ptr() if workspace is not None else None
        wb = workspace.numel() * workspace.element_size() if workspace is not None else 0
        rlx_allreduce_tree(x.data_ptr(), out.data_ptr(), count, stride, n, d, w, RLX_SUM, wp, wb,
                           _stream())
    elif algo == "tree_fused":
        if workspace is None:
            workspace = fused_tree_workspace(x, wire)
        if status is not None and (status.dtype != torch.int32 or not status.is_cuda):
            raise ValueError("status must be an int32 CUDA tensor")
        rlx_allreduce_tree_fused(x.data_ptr(), out.data_ptr(), count, stride, n, d, w, RLX_SUM,
                                 workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                 status.data_ptr() if status is not None else None, wait_limit_ns,
                                 _stream())
    else:
        raise ValueError("algo must be 'flat', 'tree' or 'tree_fused'")
    return out


def reduce_scatter(x: torch.Tensor, wire: str | None = None, out: torch.Tensor | None = None):
    """x [N, N*m] -> [N, m]: rank r gets the SUM over ranks of chunk r."""
    n, per, stride = _rows(x)
    if n == 0 or per % n:
        raise ValueError("each rank must hold N equal chunks")
    m = per // n
    out = torch.empty((n, m), dtype=x.dtype, device=x.device) if out is None else out
    rlx_reduce_scatter(x.data_ptr(), stride, out.data_ptr(), _rows(out)[2], m, n, _dtype(x),
                       _wire(wire), RLX_SUM, _stream())
    return out


def all_gather(x: torch.Tensor, wire: str | None = None, out: torch.Tensor | None = None):
    """x [N, m] -> [N, N*m]: every rank gets every rank's chunk."""
    n, m, stride = _rows(x)
    out = torch.empty((n, n * m), dtype=x.dtype, device=x.device) if out is None else out
    rlx_all_gather(x.data_ptr(), stride, out.data_ptr(), _rows(out)[2], m, n, _dtype(x),
                   _wire(wire), _stream())
    return out


def alltoall(x: torch.Tensor, wire: str | None = None, out: torch.Tensor | None = None):
    """x [N, N*m] -> [N, N*m]: chunk r of rank s lands at chunk s of rank r."""
    n, per, stride = _rows(x)
    if n == 0 or per % n:
        raise ValueError("each rank must hold N equal chunks")
    m = per // n
    out = torch.empty((n, n * m), dtype=x.dtype, device=x.device) if out is None else out
    rlx_alltoall(x.data_ptr(), stride, out.data_ptr(), _rows(out)[2], m, n, _dtype(x),
                 _wire(wire), _stream())
    return out


def quantize_fp8(x: torch.Tensor):
    """x [rows, n] fp32/bf16 -> (codes uint8 [rows, n], scales fp32 [rows, ceil(n/128)])."""
    x2 = x.reshape(x.shape[0], -1) if x.dim() != 2 else x
    rows, n, stride = _rows(x2)
    codes = torch.empty((rows, stride), dtype=torch.uint8, device=x.device)
    scales = torch.empty((rows, (n + RLX_BLOCK - 1) // RLX_BLOCK), dtype=torch.float32,
                         device=x.device)
    rlx_quantize_fp8(x2.data_ptr(), _dtype(x2), rows, n, stride, codes.data_ptr(),
                     scales.data_ptr(), _stream())
    return codes[:, :n], scales


def dequantize_fp8(codes: torch.Tensor, scales: torch.Tensor, dtype=torch.float32):
    """Inverse of quantize_fp8 for [rows, n] codes."""
    rows, n = codes.shape
    stride = codes.stride(0)
    y = torch.empty((rows, stride), dtype=dtype, device=codes.device)
    d = RLX_F32 if dtype == torch.float32 else RLX_BF16
    rlx_dequantize_fp8(codes.data_ptr(), scales.data_ptr(), rows, n, stride, y.data_ptr(), d,
                       _stream())
    return y[:, :n]
