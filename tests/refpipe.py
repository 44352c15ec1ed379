"""Independent restatements used to pin the oracle (test-side only).

Nothing here shares code with the oracle's C source or with the CUDA library.
The block quantiser below uses different machinery on purpose: fp64 numpy
division (double rounding binary64 -> binary32 is innocuous for one division,
since 53 >= 2*24 + 2) and torch's own float8_e4m3fn conversion (round to
nearest even; it agrees with a saturating encoder wherever |v| < 464).
"""
from __future__ import annotations

import numpy as np
import torch

BLOCK = 128


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_torch(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def e4m3_decode_torch(codes: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8))
    return t.view(torch.float8_e4m3fn).to(torch.float32).numpy()


def e4m3_encode_torch(v: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def quant_segment(x: np.ndarray):
    """1-D fp32 segment -> (codes, scales, dequantised fp32), 128-blocks from x[0]."""
    x = np.asarray(x, dtype=np.float32)
    n = x.size
    nb = (n + BLOCK - 1) // BLOCK
    pad = np.zeros(nb * BLOCK, dtype=np.float32)
    pad[:n] = x
    blocks = pad.reshape(nb, BLOCK).astype(np.float64)
    amax = np.abs(blocks).max(axis=1)
    s32 = (amax / 448.0).astype(np.float32)
    s64 = s32.astype(np.float64)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        q64 = np.where(s64 == 0, np.copysign(0.0, blocks), blocks / np.where(s64 == 0, 1.0, s64))
    q32 = q64.astype(np.float32)
    assert np.all(np.abs(q32) < 464.0)
    codes = e4m3_encode_torch(q32.ravel()).reshape(nb, BLOCK)
    vals = e4m3_decode_torch(codes.ravel()).reshape(nb, BLOCK).astype(np.float64)
    deq = (vals * s64).astype(np.float32)   # exact product in fp64, one rounding
    return codes.ravel()[:n], s32, deq.ravel()[:n]


def wire(x: np.ndarray, fp8: bool) -> np.ndarray:
    """What a receiver holds after segment x crossed the wire."""
    x = np.asarray(x, dtype=np.float32)
    return quant_segment(x)[2] if fp8 else x.copy()


def ordered_sum(terms) -> np.ndarray:
    """fp32 sum of the terms in the given order, starting from the first term."""
    acc = np.array(terms[0], dtype=np.float32, copy=True)
    for t in terms[1:]:
        acc = (acc + np.asarray(t, dtype=np.float32)).astype(np.float32)
    return acc


def same_bits(a, b) -> bool:
    """Bitwise equality (so +0 and -0 differ, and NaN payloads count)."""
    a, b = np.ascontiguousarray(a), np.ascontiguousarray(b)
    if a.shape != b.shape or a.dtype.itemsize != b.dtype.itemsize:
        return False
    u = {1: np.uint8, 2: np.uint16, 4: np.uint32, 8: np.uint64}[a.dtype.itemsize]
    return bool(np.array_equal(a.view(u), b.view(u)))
