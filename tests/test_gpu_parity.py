"""GPU parity: every C-ABI entry point against the CPU oracle, element by
element, on the same seeded inputs.

Bar (written here, applied everywhere): FP8 codes, scales, copied bytes and
FP32/BF16 sums are BIT-IDENTICAL to the oracle (both sides sum in rank order
with one IEEE rounding per step, so no tolerance is needed; the 1-ulp
allowance for fp32 sums is not used).  Sizes span several 128-element blocks,
partial blocks, vector tails and strides that force the element-wise kernels.
Every output sits between canary guard bands that must survive the call.
"""
import numpy as np
import pytest
import torch

import oracle
import refpipe
from gpuutil import Guarded, dcode, guarded_from, stream, to_dev, to_host
from precision_collective_reduction_fp32_b200 import binding as B
from precision_collective_reduction_fp32_b200 import build as rlx_build
from precision_collective_reduction_fp32_b200 import synth

pytestmark = pytest.mark.gpu

ORC_WIRE = {B.RLX_WIRE_NATIVE: oracle.NATIVE, B.RLX_WIRE_FP8_E4M3: oracle.FP8}
WIRES = [B.RLX_WIRE_NATIVE, B.RLX_WIRE_FP8_E4M3]
DTYPES = ["f32", "bf16"]
TDT = {"f32": torch.float32, "bf16": torch.bfloat16}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    rlx_build.build()
    oracle.build()
    B.lib()


def _sync():
    torch.cuda.synchronize()


def _bits_equal(a, b):
    return refpipe.same_bits(a, b)


# ----------------------------------------------------------------- quantiser

QN = [1, 7, 127, 128, 129, 200, 1000, 4099, 128 * 300 + 5]


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("n", QN)
@pytest.mark.parametrize("layout", ["packed", "padded", "unaligned"])
def test_quantize_dequantize(dtype, n, layout):
    rows = 3
    stride = {"packed": n, "padded": n + 3, "unaligned": n + 1}[layout]
    x = synth.rank_buffers(4, count=n, nranks=rows, stride=stride, dtype=dtype)
    off = 1 if layout == "unaligned" else 0
    gx = guarded_from(x, off)
    codes = Guarded((rows, stride), torch.uint8, off)
    nb = (n + 127) // 128
    scales = Guarded((rows, nb), torch.float32)
    B.rlx_quantize_fp8(gx.ptr(), dcode(x), rows, n, stride, codes.ptr(), scales.ptr(), stream())
    y = Guarded((rows, stride), TDT[dtype], off, fill=torch.zeros((rows, stride), dtype=TDT[dtype]))
    B.rlx_dequantize_fp8(codes.ptr(), scales.ptr(), rows, n, stride, y.ptr(), dcode(x), stream())
    _sync()
    oc, os_ = oracle.quantize(x, n=n)
    assert _bits_equal(to_host(codes.t)[:, :n], oc[:, :n])
    assert _bits_equal(to_host(scales.t), os_)
    oy = oracle.dequantize(oc, os_, n=n, dtype=x.dtype)
    assert _bits_equal(to_host(y.t)[:, :n], oy[:, :n])
    assert all(g.guards_intact() for g in (gx, codes, scales, y))


def test_quantize_special_blocks():
    x = np.zeros((1, 5 * 128 + 17), dtype=np.float32)
    x[0, 1] = -0.0
    x[0, 128:256] = np.float32(1e-44) * np.sign(np.arange(128) - 63.5).astype(np.float32)
    x[0, 256:384] = np.float32(3e-37)
    x[0, 300] = -np.float32(3e-37)
    x[0, 384:512] = np.linspace(-5, 5, 128, dtype=np.float32)
    x[0, 512:640] = np.float32(448.0) * np.linspace(-1, 1, 128, dtype=np.float32)
    x[0, 640:] = np.float32(-2.5)
    n = x.shape[1]
    codes = torch.empty((1, n), dtype=torch.uint8, device="cuda")
    scales = torch.empty((1, 6), dtype=torch.float32, device="cuda")
    B.rlx_quantize_fp8(to_dev(x).data_ptr(), B.RLX_F32, 1, n, n, codes.data_ptr(), scales.data_ptr(),
                       stream())
    _sync()
    oc, os_ = oracle.quantize(x)
    assert _bits_equal(to_host(codes), oc) and _bits_equal(to_host(scales), os_)


def test_e4m3_hardware_conversion_band():
    """Every fp32 magnitude in [2^-12, 448], both signs, through the quantiser
    with a block scale of exactly 1 (each 128-block holds 448 as its amax and
    127 test values), against the oracle's encoder."""
    lo, hi = 0x39800000, 0x43E00001
    vals = np.arange(lo, hi, dtype=np.uint32).view(np.float32)
    step = 127 * (1 << 17)
    for start in range(0, vals.size, step):
        v = vals[start:start + step]
        nblk = (v.size + 126) // 127
        for sign in (1.0, -1.0):
            blk = np.zeros((nblk, 128), dtype=np.float32)
            blk[:, 0] = 448.0
            flat = blk[:, 1:].reshape(-1)
            flat[:v.size] = v * np.float32(sign)
            blk[:, 1:] = flat.reshape(nblk, 127)
            x = blk.reshape(1, -1)
            dx = to_dev(x)
            codes = torch.empty(x.shape, dtype=torch.uint8, device="cuda")
            scales = torch.empty((1, nblk), dtype=torch.float32, device="cuda")
            B.rlx_quantize_fp8(dx.data_ptr(), B.RLX_F32, 1, x.shape[1], x.shape[1],
                               codes.data_ptr(), scales.data_ptr(), stream())
            _sync()
            assert bool((scales == 1.0).all())
            got = to_host(codes).reshape(nblk, 128)[:, 1:].reshape(-1)[:v.size]
            first = int(v[0:1].view(np.uint32)[0]) | (0x80000000 if sign < 0 else 0)
            ref = oracle.e4m3_encode_bits_range(first, v.size)
            assert _bits_equal(got, ref), hex(first)


def test_e4m3_hardware_conversion_below_band():
    """Every fp32 magnitude below 2^-12 (subnormals included), both signs,
    through the quantiser with block scale 1: the oracle maps all of them to
    a signed zero (pinned against torch and brute force); the GPU must give
    0x00 / 0x80 for every one, the oracle's code, checked here on runs spread
    over the range."""
    hi = 0x39800000
    step = 127 * (1 << 17)
    for sign_bit in (0, 0x80000000):
        for start in range(0, hi, step):
            n = min(step, hi - start)
            nblk = (n + 126) // 127
            bits = torch.arange(start, start + nblk * 127, dtype=torch.int64, device="cuda")
            bits = torch.where(bits < start + n, bits, torch.zeros_like(bits)) | sign_bit
            vals = (bits - (1 << 32) if sign_bit else bits).to(torch.int32).view(torch.float32)
            blk = torch.empty((nblk, 128), dtype=torch.float32, device="cuda")
            blk[:, 0] = 448.0
            blk[:, 1:] = vals.view(nblk, 127)
            codes = torch.empty((1, nblk * 128), dtype=torch.uint8, device="cuda")
            scales = torch.empty((1, nblk), dtype=torch.float32, device="cuda")
            B.rlx_quantize_fp8(blk.data_ptr(), B.RLX_F32, 1, nblk * 128, nblk * 128,
                               codes.data_ptr(), scales.data_ptr(), stream())
            torch.cuda.synchronize()
            assert bool((scales == 1.0).all())
            body = codes.view(nblk, 128)[:, 1:]
            assert bool((body == (0x80 if sign_bit else 0)).all()), hex(start | sign_bit)
        # the value the GPU is held to is the oracle's: runs of the same range
        for first in range(0, hi, hi // 16):
            ref = oracle.e4m3_encode_bits_range(sign_bit | first, 1 << 16)
            assert bool((ref == (0x80 if sign_bit else 0)).all())


# ------------------------------------------------------------------ allreduce

AR_CASES = [(n, c) for n in (2, 3, 8) for c in (1, 7, 127, 128, 129, 1000, 3 * 128 * 8 + 5)] + \
           [(4, 4096), (5, 1003), (16, 2000), (12, 3005), (8, 65536 + 4), (8, 128 * 1024 + 3)]


def _run_allreduce(algo, x, count, stride, wire, inplace=False, offset=0):
    n = x.shape[0]
    gs = guarded_from(x, offset)
    if inplace:
        gr = gs
    else:
        gr = Guarded(x.shape, gs.t.dtype, offset, fill=torch.zeros(x.shape, dtype=gs.t.dtype))
    if algo == "flat":
        B.rlx_allreduce_flat(gs.ptr(), gr.ptr(), count, stride, n, dcode(x), wire, B.RLX_SUM,
                             stream())
        ws = None
    else:
        need = B.rlx_workspace_bytes(B.RLX_COLL_ALLREDUCE_TREE, count, n, dcode(x), wire)
        ws = Guarded((max(need, 1),), torch.uint8) if need else None
        B.rlx_allreduce_tree(gs.ptr(), gr.ptr(), count, stride, n, dcode(x), wire, B.RLX_SUM,
                             ws.ptr() if ws else None, need, stream())
    _sync()
    assert gs.guards_intact() and gr.guards_intact() and (ws is None or ws.guards_intact())
    return to_host(gr.t)


@pytest.mark.parametrize("algo", ["flat", "tree"])
@pytest.mark.parametrize("wire", WIRES)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("nranks,count", AR_CASES)
def test_allreduce(algo, wire, dtype, nranks, count):
    for stride, off in ((count, 0), (count + 3, 0), ((count + 7) // 8 * 8, 0), (count, 1)):
        x = synth.rank_buffers(4, count=count, nranks=nranks, stride=stride, dtype=dtype)
        got = _run_allreduce(algo, x, count, stride, wire, offset=off)
        fn = oracle.allreduce_flat if algo == "flat" else oracle.allreduce_tree
        ref = fn(x, wire=ORC_WIRE[wire], count=count)
        assert _bits_equal(got[:, :count], ref[:, :count]), (stride, off)
        assert not got[:, count:].any()       # padding columns untouched (zero-filled output)


@pytest.mark.parametrize("algo", ["flat", "tree"])
@pytest.mark.parametrize("wire", WIRES)
@pytest.mark.parametrize("dtype", DTYPES)
def test_allreduce_inplace(algo, wire, dtype):
    x = synth.rank_buffers(4, count=3000, nranks=8, dtype=dtype)
    got = _run_allreduce(algo, x, 3000, 3000, wire, inplace=True)
    fn = oracle.allreduce_flat if algo == "flat" else oracle.allreduce_tree
    assert _bits_equal(got, fn(x, wire=ORC_WIRE[wire]))


@pytest.mark.parametrize("wire", WIRES)
@pytest.mark.parametrize("count,inplace", [(524_288, True), (600_003, False)])
def test_tree_in_place_mid_size(wire, count, inplace):
    """DDA-tree at a few MiB per rank, in place and not: pass 2 re-reads rows
    pass 1 streamed as input and just rewrote (read through L2 only)."""
    x = synth.rank_buffers(4, count=count, nranks=8)
    got = _run_allreduce("tree", x, count, count, wire, inplace=inplace)
    assert _bits_equal(got, oracle.allreduce_tree(x, wire=ORC_WIRE[wire]))


@pytest.mark.parametrize("wire", WIRES)
@pytest.mark.parametrize("dtype,count", [(None, 4_194_304 + 77), ("bf16", 8_388_608 + 2 * 128 + 77)])
@pytest.mark.parametrize("inplace", [False, True])
def test_tree_two_launch_ragged(wire, dtype, count, inplace):
    """Counts past the range of the one-launch cluster path, so the DDA-tree
    runs as its two launches, with a partial last block, in place and not
    (the parity cases above are small enough for the cluster path)."""
    x = synth.rank_buffers(4, count=count, nranks=8, dtype=dtype)
    got = _run_allreduce("tree", x, count, count, wire, inplace=inplace)
    assert _bits_equal(got, oracle.allreduce_tree(x, wire=ORC_WIRE[wire]))


@pytest.mark.parametrize("algo", ["flat", "tree"])
def test_bf16_fp8_large_ragged(algo):
    """bf16 on the FP8 wire past the small-message threshold (>= 32768 blocks,
    the multi-unit-per-warp launch) with an odd block count and a partial last
    block, so the last two-block unit holds one partial block."""
    count = 4_194_304 + 2 * 128 + 77
    x = synth.rank_buffers(4, count=count, nranks=8, dtype="bf16")
    got = _run_allreduce(algo, x, count, count, B.RLX_WIRE_FP8_E4M3)
    fn = oracle.allreduce_flat if algo == "flat" else oracle.allreduce_tree
    assert _bits_equal(got, fn(x, wire=oracle.FP8))


def test_bf16_fp8_reduce_scatter_large_ragged():
    """Reduce-scatter, bf16 on the FP8 wire: chunks of an odd number of
    blocks with a partial last block, past the small-message threshold."""
    n, m = 8, 524_288 + 128 + 5
    x = synth.rank_buffers(5, count=n * m, nranks=n, dtype="bf16")
    got = _chunked("rlx_reduce_scatter", x, m, n * m, m, m, B.RLX_WIRE_FP8_E4M3)
    assert _bits_equal(got, oracle.reduce_scatter(x, m, wire=oracle.FP8, recv_stride=m))


@pytest.mark.parametrize("algo", ["flat", "tree"])
@pytest.mark.parametrize("wire", WIRES)
@pytest.mark.parametrize("dtype", DTYPES)
def test_one_rank_copies(algo, wire, dtype):
    x = synth.rank_buffers(5, count=1001, nranks=1, dtype=dtype)
    assert _bits_equal(_run_allreduce(algo, x, 1001, 1001, wire), x)


@pytest.mark.parametrize("algo", ["flat", "tree"])
@pytest.mark.parametrize("wire", WIRES)
@pytest.mark.parametrize("dtype", DTYPES)
def test_worked_example(algo, wire, dtype):
    """Rank r holds torch.full((10, 20), r); every result is N(N-1)/2."""
    for nranks in (2, 3, 8, 16):
        x = synth.full_rank_values(nranks, 200, dtype)
        got = refpipe.bf16_to_f32(_run_allreduce(algo, x, 200, 200, wire)) if dtype == "bf16" \
            else _run_allreduce(algo, x, 200, 200, wire)
        assert np.all(got == nranks * (nranks - 1) / 2)


@pytest.mark.parametrize("algo", ["flat", "tree"])
@pytest.mark.parametrize("dtype", DTYPES)
def test_allreduce_fp8_special_scales(algo, dtype):
    """FP8 wire with ranks whose blocks take every scale path: all zeros
    (scale 0), ordinary values, values so small that the scale is below the
    fast-quotient bound (IEEE division), subnormal inputs, and huge values;
    units mix fast and slow blocks, and later columns make some units all fast."""
    n, count = 6, 5 * 256 + 77
    x = synth.rank_buffers(4, count=count, nranks=n).astype(np.float64)
    x[0] = 0.0
    x[2] *= 1e-30
    x[3] *= 1e-39
    x[4] *= 1e30
    x[5, :600] *= 1e-33
    x = x.astype(np.float32)
    if dtype == "bf16":
        x = synth.as_bf16_bits(x)
    got = _run_allreduce(algo, x, count, count, B.RLX_WIRE_FP8_E4M3)
    fn = oracle.allreduce_flat if algo == "flat" else oracle.allreduce_tree
    assert _bits_equal(got, fn(x, wire=oracle.FP8))


def test_signed_zero():
    x = np.full((3, 130), -0.0, dtype=np.float32)
    for algo in ("flat", "tree"):
        for wire in WIRES:
            got = _run_allreduce(algo, x, 130, 130, wire)
            assert np.all(got.view(np.uint32) == 0x80000000)


# ---------------------------------------------------- RS / AG / alltoall

CH_CASES = [(2, 1), (3, 7), (8, 128), (8, 129), (5, 300), (16, 256), (8, 4096 + 4), (4, 1)]


def _chunked(name, x, m, sstride, rstride, rlen, wire, off=0):
    n = x.shape[0]
    gs = guarded_from(x, off)
    gr = Guarded((n, rstride), gs.t.dtype, off, fill=torch.zeros((n, rstride), dtype=gs.t.dtype))
    fn = getattr(B, name)
    if name == "rlx_reduce_scatter":
        fn(gs.ptr(), sstride, gr.ptr(), rstride, m, n, dcode(x), wire, B.RLX_SUM, stream())
    else:
        fn(gs.ptr(), sstride, gr.ptr(), rstride, m, n, dcode(x), wire, stream())
    _sync()
    assert gs.guards_intact() and gr.guards_intact()
    return to_host(gr.t)


@pytest.mark.parametrize("wire", WIRES)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("nranks,m", CH_CASES)
def test_reduce_scatter(wire, dtype, nranks, m):
    for pad, off in ((0, 0), (4, 0), (1, 1)):
        x = synth.rank_buffers(5, count=nranks * m, nranks=nranks, stride=nranks * m + pad, dtype=dtype)
        got = _chunked("rlx_reduce_scatter", x, m, nranks * m + pad, m + pad, m, wire, off)
        ref = oracle.reduce_scatter(x, m, wire=ORC_WIRE[wire], recv_stride=m + pad)
        assert _bits_equal(got, ref), (pad, off)


@pytest.mark.parametrize("wire", WIRES)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("nranks,m", CH_CASES)
def test_all_gather(wire, dtype, nranks, m):
    for pad, off in ((0, 0), (4, 0), (1, 1)):
        x = synth.rank_buffers(5, count=m, nranks=nranks, stride=m + pad, dtype=dtype)
        got = _chunked("rlx_all_gather", x, m, m + pad, nranks * m + pad, nranks * m, wire, off)
        ref = oracle.all_gather(x, m, wire=ORC_WIRE[wire], recv_stride=nranks * m + pad)
        assert _bits_equal(got, ref), (pad, off)


@pytest.mark.parametrize("wire", WIRES)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("nranks,m", CH_CASES)
def test_alltoall(wire, dtype, nranks, m):
    for pad, off in ((0, 0), (4, 0), (1, 1)):
        x = synth.rank_buffers(5, count=nranks * m, nranks=nranks, stride=nranks * m + pad, dtype=dtype)
        got = _chunked("rlx_alltoall", x, m, nranks * m + pad, nranks * m + pad, nranks * m, wire, off)
        ref = oracle.alltoall(x, m, wire=ORC_WIRE[wire], recv_stride=nranks * m + pad)
        assert _bits_equal(got, ref), (pad, off)


@pytest.mark.parametrize("name", ["rlx_all_gather", "rlx_alltoall"])
@pytest.mark.parametrize("m", [8192 + 256, 3 * 1024 + 8])
def test_bf16_fp8_gathers_wide(name, m):
    """bf16 on the FP8 wire with whole 8-block units and 16-byte aligned rows
    (block pairs read and written as 16-byte pieces), a ragged last unit, and
    the same shapes on rows that are not 16-byte aligned."""
    n = 8
    for pad, off in ((0, 0), (8, 0), (4, 0), (0, 1)):   # 16-byte, 16-byte, 8-byte, 2-byte rows
        if name == "rlx_all_gather":
            x = synth.rank_buffers(5, count=m, nranks=n, stride=m + pad, dtype="bf16")
            got = _chunked(name, x, m, m + pad, n * m + pad, n * m, B.RLX_WIRE_FP8_E4M3, off)
            ref = oracle.all_gather(x, m, wire=oracle.FP8, recv_stride=n * m + pad)
        else:
            x = synth.rank_buffers(5, count=n * m, nranks=n, stride=n * m + pad, dtype="bf16")
            got = _chunked(name, x, m, n * m + pad, n * m + pad, n * m, B.RLX_WIRE_FP8_E4M3, off)
            ref = oracle.alltoall(x, m, wire=oracle.FP8, recv_stride=n * m + pad)
        assert _bits_equal(got, ref), (pad, off)


def test_torch_level_api_matches_c_abi():
    import precision_collective_reduction_fp32_b200 as rlx
    x = synth.rank_buffers(4, count=4096, nranks=8)
    dx = to_dev(x)
    for algo in ("flat", "tree"):
        for wire in ("native", "fp8"):
            y = rlx.allreduce(dx, algo=algo, wire=wire)
            ref = (oracle.allreduce_flat if algo == "flat" else oracle.allreduce_tree)(
                x, wire=oracle.FP8 if wire == "fp8" else oracle.NATIVE)
            torch.cuda.synchronize()
            assert _bits_equal(to_host(y), ref)
    c, s = rlx.quantize_fp8(dx)
    oc, os_ = oracle.quantize(x)
    torch.cuda.synchronize()
    assert _bits_equal(to_host(c), oc) and _bits_equal(to_host(s), os_)
