"""CPU oracle for the emulated RCCLX collectives -- TEST INFRASTRUCTURE ONLY.

Only the test-suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg may import this package.  The library under
``precision_collective_reduction_fp32_b200`` never imports it, and this package
imports nothing from the library: the two share no code.

The arithmetic lives in ``oracle.c`` (plain single-threaded C, compiled with
``-O2 -ffp-contract=off``); this module only compiles it and passes numpy
arrays to it.  Rank buffers are 2-D numpy arrays ``[nranks, stride]`` of
``float32`` (fp32) or ``uint16`` (bf16 bit patterns).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F32, BF16 = 0, 1
NATIVE, FP8 = 0, 1
BLOCK = 128

CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-std=c99"]


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (if stale or missing)."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "oracle.h")))
    if force or stale:
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        # ORACLE_LIB lets the oracle's own mutation test load a deliberately
        # broken build of oracle.c; nothing else sets it.
        L = ctypes.CDLL(os.environ.get("ORACLE_LIB") or build())
        P, S, I, U8, U32, F = (ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int,
                               ctypes.c_uint8, ctypes.c_uint32, ctypes.c_float)
        L.orc_e4m3_value.argtypes, L.orc_e4m3_value.restype = [U8], F
        L.orc_e4m3_encode.argtypes, L.orc_e4m3_encode.restype = [F], U8
        L.orc_e4m3_encode_bits_range.argtypes, L.orc_e4m3_encode_bits_range.restype = [U32, S, P], None
        L.orc_bf16_to_f32.argtypes, L.orc_bf16_to_f32.restype = [ctypes.c_uint16], F
        L.orc_f32_to_bf16.argtypes, L.orc_f32_to_bf16.restype = [F], ctypes.c_uint16
        L.orc_quantize.argtypes, L.orc_quantize.restype = [I, P, S, S, S, P, P], I
        L.orc_dequantize.argtypes, L.orc_dequantize.restype = [P, P, S, S, S, I, P], I
        for name in ("orc_allreduce_flat", "orc_allreduce_tree"):
            fn = getattr(L, name)
            fn.argtypes, fn.restype = [I, I, P, P, S, S, I], I
        for name in ("orc_reduce_scatter", "orc_all_gather", "orc_alltoall"):
            fn = getattr(L, name)
            fn.argtypes, fn.restype = [I, I, P, S, P, S, S, I], I
        L.orc_tree_chunk.argtypes, L.orc_tree_chunk.restype = [S, I], S
        _lib = L
    return _lib


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError("rank buffers are float32 or uint16 (bf16 bits), got %s" % a.dtype)


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError("oracle %s rejected its input (rc=%d)" % (what, rc))


# ----------------------------------------------------------------- codecs

def e4m3_value(code: int) -> float:
    return float(lib().orc_e4m3_value(int(code)))


def e4m3_encode(v: float) -> int:
    return int(lib().orc_e4m3_encode(float(v)))


def e4m3_encode_bits_range(first: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint8)
    lib().orc_e4m3_encode_bits_range(first, n, _ptr(out))
    return out


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32).ravel()
    return np.array([lib().orc_f32_to_bf16(float(v)) for v in x], dtype=np.uint16)


def nblocks(n: int) -> int:
    return (n + BLOCK - 1) // BLOCK


def quantize(x: np.ndarray, n: int | None = None):
    """x: [rows, stride] -> (codes uint8 [rows, stride], scales f32 [rows, nblocks(n)])."""
    x = np.ascontiguousarray(x)
    if x.ndim == 1:
        x = x[None, :]
    rows, stride = x.shape
    n = stride if n is None else n
    codes = np.zeros((rows, stride), dtype=np.uint8)
    scales = np.zeros((rows, nblocks(n)), dtype=np.float32)
    _check(lib().orc_quantize(_dtype_code(x), _ptr(x), rows, n, stride, _ptr(codes), _ptr(scales)),
           "quantize")
    return codes, scales


def dequantize(codes: np.ndarray, scales: np.ndarray, n: int | None = None, dtype=np.float32):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    if codes.ndim == 1:
        codes, scales = codes[None, :], scales.reshape(1, -1)
    rows, stride = codes.shape
    n = stride if n is None else n
    y = np.zeros((rows, stride), dtype=dtype)
    _check(lib().orc_dequantize(_ptr(codes), _ptr(scales), rows, n, stride,
                                _dtype_code(y), _ptr(y)), "dequantize")
    return y


# ------------------------------------------------------------ collectives

def _allreduce(fn, x: np.ndarray, wire: int, count: int | None, out: np.ndarray | None):
    x = np.ascontiguousarray(x)
    nranks, stride = x.shape
    count = stride if count is None else count
    y = np.zeros_like(x) if out is None else out
    _check(fn(_dtype_code(x), wire, _ptr(x), _ptr(y), count, stride, nranks), fn.__name__)
    return y


def allreduce_flat(x: np.ndarray, wire: int = NATIVE, count: int | None = None, out=None):
    return _allreduce(lib().orc_allreduce_flat, x, wire, count, out)


def allreduce_tree(x: np.ndarray, wire: int = NATIVE, count: int | None = None, out=None):
    return _allreduce(lib().orc_allreduce_tree, x, wire, count, out)


def tree_chunk(count: int, nranks: int) -> int:
    return int(lib().orc_tree_chunk(count, nranks))


def reduce_scatter(x: np.ndarray, m: int, wire: int = NATIVE, recv_stride: int | None = None):
    x = np.ascontiguousarray(x)
    nranks, sstride = x.shape
    rstride = m if recv_stride is None else recv_stride
    y = np.zeros((nranks, rstride), dtype=x.dtype)
    _check(lib().orc_reduce_scatter(_dtype_code(x), wire, _ptr(x), sstride, _ptr(y), rstride,
                                    m, nranks), "reduce_scatter")
    return y


def all_gather(x: np.ndarray, m: int, wire: int = NATIVE, recv_stride: int | None = None):
    x = np.ascontiguousarray(x)
    nranks, sstride = x.shape
    rstride = nranks * m if recv_stride is None else recv_stride
    y = np.zeros((nranks, rstride), dtype=x.dtype)
    _check(lib().orc_all_gather(_dtype_code(x), wire, _ptr(x), sstride, _ptr(y), rstride,
                                m, nranks), "all_gather")
    return y


def alltoall(x: np.ndarray, m: int, wire: int = NATIVE, recv_stride: int | None = None):
    x = np.ascontiguousarray(x)
    nranks, sstride = x.shape
    rstride = nranks * m if recv_stride is None else recv_stride
    y = np.zeros((nranks, rstride), dtype=x.dtype)
    _check(lib().orc_alltoall(_dtype_code(x), wire, _ptr(x), sstride, _ptr(y), rstride,
                              m, nranks), "alltoall")
    return y
