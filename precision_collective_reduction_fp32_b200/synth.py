"""Seeded synthetic rank buffers for the emulated collectives.

This module only draws numbers: it holds none of the collectives' arithmetic,
and both the CUDA library's tests and the CPU oracle's tests take their inputs
from it.  Every draw comes from a CPU ``torch.Generator`` seeded with
``1000 * workload + rank``, so the same (workload, rank, size) always gives the
same bytes.  bf16 workloads are drawn in fp32 and rounded by torch's own
``.to(torch.bfloat16)``.

Workloads (N simulated ranks, one row each; the shapes are those of the
prefill / decode messages and the >= 16 MB low-precision messages the RCCLX
pages talk about):

  1  tiny      N=8, fp32 [10, 20] = 200 elements, N(0, 1)
  2  decode    N=8, bf16 [32, 8192] = 262,144 elements (512 KiB / rank), N(0, 0.5)
  3  prefill   N=8, bf16 [4096, 8192] = 33,554,432 elements (64 MiB / rank), N(0, 1)
  4  lp-ar     N=8, fp32 [16,777,216] (64 MiB / rank), N(0, 1) with each element
               independently multiplied by 100 with probability 0.01 (outliers)
  5  lp-coll   N=8, fp32 [67,108,864] (256 MiB / rank), Student-t with 3 degrees
               of freedom, t = z / sqrt(chi2_3 / 3)
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    key: int
    name: str
    nranks: int
    count: int          # elements per rank
    dtype: str          # "f32" or "bf16"
    dist: str           # "normal", "normal_outliers", "student_t3"
    std: float = 1.0
    op: str = ""        # the collective this workload is quoted on

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2


WORKLOADS = {
    1: Workload(1, "tiny", 8, 200, "f32", "normal", 1.0,
                "DDA-flat allreduce, fp32 and FP8 wire"),
    2: Workload(2, "decode", 8, 32 * 8192, "bf16", "normal", 0.5,
                "DDA-flat allreduce, bf16, fp32 accumulation"),
    3: Workload(3, "prefill", 8, 4096 * 8192, "bf16", "normal", 1.0,
                "DDA-tree allreduce (reduce-scatter pass + all-gather pass), bf16"),
    4: Workload(4, "lp-allreduce", 8, 16_777_216, "f32", "normal_outliers", 1.0,
                "FP8-wire allreduce (fused dequantise-sum-requantise)"),
    5: Workload(5, "lp-collectives", 8, 67_108_864, "f32", "student_t3", 1.0,
                "FP8-wire reduce-scatter, all-gather and alltoall"),
}


def seed(workload: int, rank: int) -> int:
    return 1000 * workload + rank


def _draw(dist: str, count: int, g: torch.Generator, std: float, device) -> torch.Tensor:
    if dist == "normal":
        x = torch.randn(count, generator=g, dtype=torch.float32, device=device) * std
    elif dist == "normal_outliers":
        x = torch.randn(count, generator=g, dtype=torch.float32, device=device) * std
        hit = torch.rand(count, generator=g, device=device) < 0.01
        x = torch.where(hit, x * 100.0, x)
    elif dist == "student_t3":
        x = torch.empty(count, dtype=torch.float32, device=device)
        step = 1 << 24
        for lo in range(0, count, step):
            n = min(step, count - lo)
            z = torch.randn(n, generator=g, dtype=torch.float64, device=device)
            c = torch.randn((3, n), generator=g, dtype=torch.float64, device=device).square().sum(0)
            x[lo:lo + n] = (z / torch.sqrt(c / 3.0)).to(torch.float32)
    else:
        raise ValueError(dist)
    return x


def draw_row(dist: str, count: int, s: int, std: float = 1.0) -> np.ndarray:
    """One rank's fp32 values."""
    return _draw(dist, count, torch.Generator().manual_seed(s), std, "cpu").numpy()


def as_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 values -> bf16 bit patterns (uint16), rounded by torch."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def rank_buffers(workload: int, count: int | None = None, nranks: int | None = None,
                 stride: int | None = None, dtype: str | None = None) -> np.ndarray:
    """[nranks, stride] host array for a workload (optionally resized).

    fp32 -> float32 array; bf16 -> uint16 array of bf16 bit patterns.  Padding
    columns past `count` hold a fixed marker value so that a kernel that reads
    or writes past the row end is seen.
    """
    w = WORKLOADS[workload]
    count = w.count if count is None else count
    nranks = w.nranks if nranks is None else nranks
    stride = count if stride is None else stride
    dtype = w.dtype if dtype is None else dtype
    if dtype == "f32":
        out = np.full((nranks, stride), np.float32(-7.25), dtype=np.float32)
    else:
        out = np.full((nranks, stride), 0xC0E8, dtype=np.uint16)  # bf16 -7.25
    for r in range(nranks):
        x = draw_row(w.dist, count, seed(workload, r), w.std)
        out[r, :count] = x if dtype == "f32" else as_bf16_bits(x)
    return out


def device_rank_buffers(workload: int, device, salt: int = 0,
                        count: int | None = None) -> torch.Tensor:
    """[nranks, count] torch tensor of a workload drawn directly on a CUDA
    device (fp32, or bf16 rounded from fp32), for timing at full size where
    the host draw would take a minute.  Same recipe as rank_buffers, drawn
    from the device's generator seeded with seed(workload, rank) + salt, so
    the values follow the same distribution but are not the host bytes."""
    w = WORKLOADS[workload]
    count = w.count if count is None else count
    out = torch.empty((w.nranks, count), dtype=torch.float32 if w.dtype == "f32"
                      else torch.bfloat16, device=device)
    for r in range(w.nranks):
        g = torch.Generator(device=device).manual_seed(seed(workload, r) + salt)
        out[r].copy_(_draw(w.dist, count, g, w.std, device))
    return out


def full_rank_values(nranks: int, count: int, dtype: str = "f32", stride: int | None = None):
    """The pages' worked example: rank r holds torch.full(shape, r)."""
    stride = count if stride is None else stride
    x = np.zeros((nranks, stride), dtype=np.float32)
    for r in range(nranks):
        x[r, :count] = float(r)
    return x if dtype == "f32" else as_bf16_bits(x)
