"""Helpers for the GPU parity tests: host<->device moves of rank buffers and
guard-banded device allocations (a canary pattern around every output that a
test checks untouched after the call)."""
from __future__ import annotations

import numpy as np
import torch

from precision_collective_reduction_fp32_b200 import binding as B

GUARD = 4096          # bytes of canary before and after each guarded buffer
CANARY = 0xA5


def dcode(a: np.ndarray) -> int:
    return B.RLX_BF16 if a.dtype == np.uint16 else B.RLX_F32


def to_dev(a: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    if a.dtype == np.uint8:
        return torch.from_numpy(a).cuda()
    return torch.from_numpy(a).cuda()


def to_host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


class Guarded:
    """A device buffer of `shape`/`dtype` with canary bytes on both sides.

    `offset_elems` shifts the start by whole elements, to reach the
    element-wise (unaligned) kernels."""

    def __init__(self, shape, dtype: torch.dtype, offset_elems: int = 0, fill=None):
        es = torch.empty((), dtype=dtype).element_size()
        n = int(np.prod(shape))
        self.lo = GUARD + offset_elems * es
        self.nbytes = n * es
        self.raw = torch.full((self.lo + self.nbytes + GUARD,), CANARY, dtype=torch.uint8,
                              device="cuda")
        self.t = self.raw[self.lo:self.lo + self.nbytes].view(dtype).view(*shape)
        if fill is not None:
            self.t.copy_(fill)

    def ptr(self) -> int:
        return self.t.data_ptr()

    def guards_intact(self) -> bool:
        head = self.raw[:self.lo]
        tail = self.raw[self.lo + self.nbytes:]
        return bool((head == CANARY).all().item()) and bool((tail == CANARY).all().item())


def guarded_from(a: np.ndarray, offset_elems: int = 0) -> Guarded:
    d = to_dev(a)
    return Guarded(a.shape, d.dtype, offset_elems, fill=d)


def stream() -> int | None:
    return torch.cuda.current_stream().cuda_stream or None
