#!/usr/bin/env python
"""Benchmark of the emulated RCCLX collectives on B200.

One STEP is one pass of every hot-path operation over one batch of N=8
simulated ranks x 16,777,216 fp32 elements (64 MiB per rank, N(0,1) with 1%
of the elements scaled x100 as outliers -- the >= 16 MB low-precision message
size the RCCLX pages target):

    quantise (128-block FP8 E4M3), DDA-flat allreduce (native fp32 wire),
    dequantise, DDA-flat allreduce (FP8 wire),
    DDA-tree allreduce    (native fp32 wire, FP8 wire: fused
                           dequantise-sum-requantise pass + all-gather pass),
    reduce-scatter, all-gather, alltoall (native and FP8 wire).

`value` is the effective HBM bandwidth of the whole step: the algorithmic
bytes of all operations (inputs read once, outputs written once, plus the
tree's wire payload written by pass 1 and read by pass 2) divided by the
device time of the timed steps.  Every operation touches >= 576 MiB, far more
than the 126 MB L2, so no flush is needed between steps; dequantise runs after
the 1 GiB DDA-flat pass, not straight after quantise, so it reads the codes
from HBM.  `roofline` is the slowest single-kernel operation against the
measured copy bandwidth, and `roofline.target` the FP8 DDA-tree allreduce
(the fused low-precision allreduce the >= 16 MB target is quoted on).
`e2e` is that one collective end to end: each step uploads the 512 MiB
input from pinned host memory, runs it and downloads the 512 MiB result, in
column ranges so that the two PCIe directions overlap.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

With --gpus N > 1 (under torchrun) each GPU runs its own independent batch:
there is no data-path exchange between GPUs (the emulated ranks all live in
one GPU's memory), so the scaling is weak and `value` sums all GPUs.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

NRANKS = 8
COUNT = 16_777_216
M = COUNT // NRANKS
BLOCK = 128
MIB = 1 << 20
WORKLOAD = 4        # seeded workload id in synth (N(0,1) + 1% x100 outliers)
CPU_SAMPLE = 8_388_608   # elements per rank in the oracle's bounded sample (~10 s)
HBM_NOMINAL_GBS = 7700.0  # B200 HBM3e, nominal (the roofline itself uses the measured copy peak)


# --------------------------------------------------------------- bytes model

def op_bytes(count: int, nranks: int, esize: int = 4) -> dict[str, int]:
    """Algorithmic HBM bytes per launch of each operation on [nranks][count]."""
    n, c, m = nranks, count, count // nranks
    nblk = (c + BLOCK - 1) // BLOCK
    codes, scales = n * c, n * nblk * 4
    data = n * c * esize
    payload = c + nblk * 4                       # tree FP8 wire payload
    return {
        "quantize_fp8": data + codes + scales,
        "dequantize_fp8": codes + scales + data,
        "allreduce_flat_native": 2 * data,
        "allreduce_flat_fp8": 2 * data,
        "allreduce_tree_native": data + c * esize + c * esize + (n - 1) * c * esize,
        "allreduce_tree_fp8": data + payload + payload + data,
        "reduce_scatter_native": data + n * m * esize,
        "reduce_scatter_fp8": data + n * m * esize,
        "all_gather_native": n * m * esize + data,
        "all_gather_fp8": n * m * esize + data,
        "alltoall_native": 2 * data,
        "alltoall_fp8": 2 * data,
    }


OPS = list(op_bytes(COUNT, NRANKS).keys())
# the operation the >= 16 MB low-precision target is quoted on
TARGET_OP = "allreduce_tree_fp8"
KERNELS_PER_OP = {op: (2 if op.startswith("allreduce_tree") else 1) for op in OPS}


# ------------------------------------------------------------ multi-GPU host

def gpu_seed(sim_rank: int, gpu_rank: int) -> int:
    """Seed of simulated rank `sim_rank` in the batch of GPU `gpu_rank`: every
    GPU works on its own independent batch (weak scaling, no exchange)."""
    from precision_collective_reduction_fp32_b200 import synth
    return synth.seed(WORKLOAD, sim_rank) + 100 * gpu_rank


def max_over_ranks(x: float, device=None) -> float:
    """The maximum of x over all processes of the default group (x itself
    when there is no group).  Timings are reported as the slowest rank."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world: int, bytes_per_step: int, steps: int, ms: float) -> float:
    """Effective GB/s of all GPUs together: every GPU moved bytes_per_step per
    step, the job took `ms` (the slowest GPU)."""
    return world * bytes_per_step * steps / (ms * 1e-3) / 1e9


# ------------------------------------------------------------------ helpers

def peaks() -> tuple[float, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


def source_hash() -> str:
    csrc = os.path.join(ROOT, "precision_collective_reduction_fp32_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(op: str, count: int = COUNT):
    """dram bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources and at this count per rank (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    e = rec.get(op)
    if not e or e.get("src_sha") != source_hash() or e.get("count") != count:
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples: list[tuple[float, int, int]] = []
        self.period = period_s
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001 -- clocks are reported as unavailable
            self.err = repr(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self, t0: float, t1: float) -> dict:
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML: " + self.err}
        self._stop.set()
        self._t.join()
        inside = [s for s in self.samples if t0 <= s[0] <= t1] or self.samples[-3:]
        mhz = [s[1] for s in inside]
        bits = 0
        for s in inside:
            bits |= s[2]
        reasons = [name for b, name in self.REASONS.items() if bits & b and name != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(inside)}


# ------------------------------------------------------------ the GPU step

class Step:
    """Device buffers for one batch and the twelve operations of one step,
    each issued through the C ABI (librlx.so) on the current stream."""

    def __init__(self, x_host: np.ndarray, device, pad: int = 0):
        import torch
        from precision_collective_reduction_fp32_b200 import binding as B
        self.B, self.torch = B, torch
        n, c = x_host.shape
        self.n, self.c, self.m = n, c, c // n
        # rank rows are `pitch` elements apart (pad > 0 breaks power-of-two
        # distances between the rows that are streamed together)
        self.pitch, self.mpitch = c + pad, self.m + pad
        t = lambda *s, dt=torch.float32: torch.empty(*s, dtype=dt, device=device)
        self.x = t((n, self.pitch))
        self.x[:, :c].copy_(torch.from_numpy(x_host))
        # two of each output, alternated so that no operation writes the
        # buffer its predecessor has just written (dirty L2 lines of one
        # operation are never overwritten by the next)
        self.out1, self.out2 = t((n, self.pitch)), t((n, self.pitch))
        self.y1, self.y2 = t((n, self.pitch)), t((n, self.pitch))
        self.out = self.out2                       # holds the FP8 tree allreduce result
        self.codes = t((n, self.pitch), dt=torch.uint8)
        self.scales = t((n, (c + BLOCK - 1) // BLOCK))
        self.rs1, self.rs2 = t((n, self.mpitch)), t((n, self.mpitch))
        self.ws_bytes = B.rlx_workspace_bytes(B.RLX_COLL_ALLREDUCE_TREE, c, n, B.RLX_F32,
                                              B.RLX_WIRE_FP8_E4M3)
        self.ws = t((self.ws_bytes,), dt=torch.uint8)

    def ops(self, stream):
        B, n, c, m, p, mp = self.B, self.n, self.c, self.m, self.pitch, self.mpitch
        x = self.x.data_ptr()
        o1, o2 = self.out1.data_ptr(), self.out2.data_ptr()
        y1, y2 = self.y1.data_ptr(), self.y2.data_ptr()
        r1, r2 = self.rs1.data_ptr(), self.rs2.data_ptr()
        F, NAT, FP8 = B.RLX_F32, B.RLX_WIRE_NATIVE, B.RLX_WIRE_FP8_E4M3
        # dequantise runs after DDA-flat, so that the 1 GiB flat pass has
        # pushed quantise's codes out of L2 before dequantise reads them
        return [
            ("quantize_fp8", lambda: B.rlx_quantize_fp8(x, F, n, c, p, self.codes.data_ptr(),
                                                        self.scales.data_ptr(), stream)),
            ("allreduce_flat_native", lambda: B.rlx_allreduce_flat(x, o1, c, p, n, F, NAT, B.RLX_SUM, stream)),
            ("dequantize_fp8", lambda: B.rlx_dequantize_fp8(self.codes.data_ptr(), self.scales.data_ptr(),
                                                            n, c, p, y2, F, stream)),
            ("allreduce_flat_fp8", lambda: B.rlx_allreduce_flat(x, o2, c, p, n, F, FP8, B.RLX_SUM, stream)),
            ("allreduce_tree_native", lambda: B.rlx_allreduce_tree(x, o1, c, p, n, F, NAT, B.RLX_SUM,
                                                                   None, 0, stream)),
            ("allreduce_tree_fp8", lambda: B.rlx_allreduce_tree(x, o2, c, p, n, F, FP8, B.RLX_SUM,
                                                                self.ws.data_ptr(), self.ws_bytes, stream)),
            ("reduce_scatter_native", lambda: B.rlx_reduce_scatter(x, p, r1, mp, m, n, F, NAT, B.RLX_SUM, stream)),
            ("reduce_scatter_fp8", lambda: B.rlx_reduce_scatter(x, p, r2, mp, m, n, F, FP8, B.RLX_SUM, stream)),
            ("all_gather_native", lambda: B.rlx_all_gather(r1, mp, y1, p, m, n, F, NAT, stream)),
            ("all_gather_fp8", lambda: B.rlx_all_gather(r2, mp, y2, p, m, n, F, FP8, stream)),
            ("alltoall_native", lambda: B.rlx_alltoall(x, p, y1, p, m, n, F, NAT, stream)),
            ("alltoall_fp8", lambda: B.rlx_alltoall(x, p, y2, p, m, n, F, FP8, stream)),
        ]


try:   # strided host<->device copies in one call (plumbing only)
    from cuda.bindings import runtime as _rt
except ImportError:
    _rt = None


class E2ETreeFp8:
    """End to end through the C ABI, one collective per step: copy the rank
    buffers from pinned host memory to the device, run the FP8 DDA-tree
    allreduce (fused dequantise-sum-requantise pass + all-gather pass) and
    copy the result back to pinned host memory.

    Each step is cut into `slices` column ranges of the [N][count] rank rows
    (multiples of the 128-element FP8 block, so every block and the result
    are those of one call on the whole rows: the tree's result does not depend
    on its chunking), and each range is uploaded, reduced by one
    rlx_allreduce_tree call on the strided rows and downloaded on its own, on
    three streams (uploads, kernels, downloads) with two device batches: the
    upload of one range overlaps the download of an earlier one, so both
    PCIe directions stay busy, and only one range's transfer is not
    overlapped at the start and end.  Calling the object with a step count
    returns the device time of those steps (ms), from the first upload's
    start to the last download's end; `result(k)` is step k's host output
    buffer."""

    def __init__(self, x_host: np.ndarray, dev, slices: int = 8):
        import torch
        from precision_collective_reduction_fp32_b200 import binding as B
        self.B, self.torch = B, torch
        self.n, self.c = x_host.shape
        while slices > 1 and (self.c % slices or (self.c // slices) % BLOCK):
            slices -= 1
        self.slices, self.w = slices, self.c // slices
        self.wsb = B.rlx_workspace_bytes(B.RLX_COLL_ALLREDUCE_TREE, self.w, self.n, B.RLX_F32,
                                         B.RLX_WIRE_FP8_E4M3)
        self.host_in = torch.from_numpy(x_host).pin_memory()
        self.host_out = [torch.empty((self.n, self.c), dtype=torch.float32).pin_memory()
                         for _ in range(2)]
        self.dx = [torch.empty((self.n, self.c), dtype=torch.float32, device=dev) for _ in range(2)]
        self.dy = [torch.empty_like(self.dx[0]) for _ in range(2)]
        self.ws = torch.empty(max(self.wsb, 1), dtype=torch.uint8, device=dev)
        self.stream = torch.cuda.current_stream(dev)
        self.s_in, self.s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        self.h2d_bytes = self.d2h_bytes = self.n * self.c * 4

    def result(self, k: int):
        return self.host_out[k % 2]

    def _copy_range(self, dst, src, lo: int, hi: int, h2d: bool, stream) -> None:
        """Columns [lo, hi) of all N rows, src -> dst (both [N][count]): one
        2-D copy (cudaMemcpy2DAsync) when cuda-python's runtime bindings are
        importable, else one copy per row."""
        if _rt is not None:
            pitch, width = self.c * 4, (hi - lo) * 4
            kind = (_rt.cudaMemcpyKind.cudaMemcpyHostToDevice if h2d
                    else _rt.cudaMemcpyKind.cudaMemcpyDeviceToHost)
            err, = _rt.cudaMemcpy2DAsync(dst[0, lo:].data_ptr(), pitch, src[0, lo:].data_ptr(), pitch,
                                         width, self.n, kind, stream.cuda_stream)
            if err != _rt.cudaError_t.cudaSuccess:
                raise RuntimeError("cudaMemcpy2DAsync failed: %s" % err)
            return
        for r in range(self.n):
            dst[r, lo:hi].copy_(src[r, lo:hi], non_blocking=True)

    def __call__(self, nsteps: int) -> float:
        torch, B = self.torch, self.B
        n, c, w, S = self.n, self.c, self.w, self.slices
        sp = self.stream.cuda_stream or None
        ev = lambda: torch.cuda.Event(enable_timing=True)
        start = ev()
        ev_in, ev_c, ev_out = ([[ev() for _ in range(S)] for _ in range(nsteps)] for _ in range(3))
        start.record(self.s_in)
        for k in range(nsteps):
            b = k % 2
            dx, dy, ho = self.dx[b], self.dy[b], self.host_out[b]
            for i in range(S):
                lo, hi = i * w, (i + 1) * w
                with torch.cuda.stream(self.s_in):
                    if k >= 2:
                        self.s_in.wait_event(ev_c[k - 2][i])    # range i of batch b is free again
                    self._copy_range(dx, self.host_in, lo, hi, True, self.s_in)
                    ev_in[k][i].record(self.s_in)
                self.stream.wait_event(ev_in[k][i])
                if k >= 2:
                    self.stream.wait_event(ev_out[k - 2][i])    # its result was read out
                B.rlx_allreduce_tree(dx[0, lo:].data_ptr(), dy[0, lo:].data_ptr(), w, c, n,
                                     B.RLX_F32, B.RLX_WIRE_FP8_E4M3, B.RLX_SUM,
                                     self.ws.data_ptr(), self.wsb, sp)   # raises on failure
                ev_c[k][i].record(self.stream)
                with torch.cuda.stream(self.s_out):
                    self.s_out.wait_event(ev_c[k][i])
                    self._copy_range(ho, dy, lo, hi, False, self.s_out)
                    ev_out[k][i].record(self.s_out)
        torch.cuda.synchronize()
        return start.elapsed_time(ev_out[-1][-1])


def run_gpu(args, rank: int, world: int) -> dict | None:
    import torch
    import torch.distributed as dist
    from precision_collective_reduction_fp32_b200 import synth

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    # each GPU gets its own independent batch (different seeds per GPU)
    count = args.count
    x_host = np.empty((NRANKS, count), dtype=np.float32)
    for r in range(NRANKS):
        x_host[r] = synth.draw_row("normal_outliers", count, gpu_seed(r, rank))
    step = Step(x_host, dev)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream or None
    ops = step.ops(sp)
    if args.only:
        ops = [(n, f) for n, f in ops if n in args.only.split(",")]
        assert ops, "unknown --only operation"
    bytes_ = {n: b for n, b in op_bytes(count, NRANKS).items() if n in dict(ops)}
    step_bytes = sum(bytes_.values())

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        for _, f in ops:
            f()
    torch.cuda.synchronize()

    # ---- device-timed region 1: K whole steps, events only at the two ends
    # (an event between two kernels would keep the second from starting
    # while the first drains), barrier + synchronize on both sides.
    K = args.steps
    clocks = ClockSampler(local)
    clocks.start()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    e_start.record(stream)
    for k in range(K):
        for _, f in ops:
            f()
    e_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    total_ms = max_over_ranks(e_start.elapsed_time(e_end), dev)

    # ---- device-timed region 2: the same K steps with an event after every
    # operation, for the per-operation times and the roofline.
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(ops) + 1)] for _ in range(K)]
    barrier()
    torch.cuda.synchronize()
    for k in range(K):
        ev[k][0].record(stream)
        for i, (_, f) in enumerate(ops):
            f()
            ev[k][i + 1].record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    barrier()
    clk = clocks.stop(t0, t1)
    per_op_ms = {name: 0.0 for name, _ in ops}
    for k in range(K):
        for i, (name, _) in enumerate(ops):
            per_op_ms[name] += ev[k][i].elapsed_time(ev[k][i + 1])
    per_op_total_ms = ev[0][0].elapsed_time(ev[K - 1][-1])

    # ---- end to end, one collective (the FP8 DDA-tree allreduce, the
    # operation the >= 16 MB target is quoted on): upload, kernels, download
    Ke = max(1, min(K, args.e2e_steps))
    if world > 1:
        # the step's buffers are no longer needed: make room on the device
        del ops, step
        torch.cuda.empty_cache()
    e2e_run = E2ETreeFp8(x_host, dev)
    e2e_run(2)
    barrier()
    e2e_ms = max_over_ranks(e2e_run(Ke), dev)
    barrier()
    e2e_slices = e2e_run.slices
    del e2e_run
    if rank != 0:
        return None

    peak, peak_kind = peaks()
    value = whole_job_gbs(world, step_bytes, K, total_ms)
    per_op = {}
    for name in per_op_ms:
        ms = per_op_ms[name] / K
        gbs = bytes_[name] / (ms * 1e-3) / 1e9
        per_op[name] = {"us": round(ms * 1e3, 2), "GB/s": round(gbs, 1),
                        "Gelem/s": round(NRANKS * count / (ms * 1e-3) / 1e9, 1),
                        "frac": round(gbs / peak, 3),
                        "frac_nominal": round(gbs / HBM_NOMINAL_GBS, 3),
                        "MiB": round(bytes_[name] / MIB, 1)}
    single = [n for n in per_op_ms if KERNELS_PER_OP[n] == 1]
    dom = max(single, key=lambda n: per_op_ms[n])
    dom_gbs = per_op[dom]["GB/s"]
    traffic = recorded_traffic(dom, count)
    peak_desc = ("%s HBM copy bandwidth (read + write bytes of a 1 GiB device copy); read-heavy "
                 "operations can exceed it, so every fraction is also given against the nominal "
                 "%.0f GB/s" % (peak_kind, HBM_NOMINAL_GBS))
    e2e_bytes = op_bytes(count, NRANKS)[TARGET_OP]
    res = {
        "metric": "emulated N=8 allreduce effective HBM GB/s (fp32 & FP8) and % of B200 HBM peak",
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / K, 4),
        "ms_per_step_with_op_events": round(per_op_total_ms / K, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {
            "workload": "N=8 simulated ranks x fp32[16,777,216] (64 MiB/rank), N(0,1) with 1% "
                        "x100 outliers; one step = quantise, DDA-flat native, dequantise, DDA-flat "
                        "FP8, DDA-tree allreduce (native and FP8 wire), reduce-scatter, all-gather, "
                        "alltoall (native and FP8 wire)",
            "nranks": NRANKS, "count": count, "elem": "fp32", "fp8": "e4m3, 128-block fp32 scales",
            "bytes_per_step": step_bytes,
            "l2": "no flush: every operation streams >= 576 MiB, > 126 MB L2; dequantise "
                  "follows the 1 GiB DDA-flat pass, not quantise",
            "parallelism": "independent batch per GPU" if world > 1 else "single GPU",
        },
        "hbm_frac": round(value / world / peak, 3),
        "hbm_frac_nominal": round(value / world / HBM_NOMINAL_GBS, 3),
        "peak_note": peak_desc,
        "ops": per_op,
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": dom_gbs, "peak": peak,
                     "unit": "GB/s", "frac": round(dom_gbs / peak, 3), "traffic": traffic,
                     "algorithmic_bytes": bytes_[dom], "peak_kind": peak_kind + " copy"},
        "gpu_launches": K * sum(KERNELS_PER_OP[n] for n in bytes_),
        "gpu_launches_breakdown_pass": K * sum(KERNELS_PER_OP[n] for n in bytes_),
        "gpu_launches_e2e": Ke * e2e_slices * KERNELS_PER_OP[TARGET_OP],
        "clocks": clk,
        "e2e": {"value": round(whole_job_gbs(world, e2e_bytes, Ke, e2e_ms), 1), "unit": "GB/s",
                "h2d_bytes_per_step": NRANKS * count * 4, "d2h_bytes_per_step": NRANKS * count * 4,
                "ms_per_step": round(e2e_ms / Ke, 3), "steps": Ke,
                "operation": TARGET_OP,
                "numerator": "the operation's algorithmic HBM bytes (%d per step)" % e2e_bytes,
                "pcie_GBs": round(world * 2 * NRANKS * count * 4 * Ke / (e2e_ms * 1e-3) / 1e9, 1),
                "overlap": "each step in %d column ranges, each uploaded, reduced by one "
                           "rlx_allreduce_tree call and downloaded; uploads, kernels and downloads "
                           "on three streams, two device batches" % e2e_slices},
    }
    if TARGET_OP in per_op:
        t = per_op[TARGET_OP]
        res["roofline"]["target"] = {
            "operation": TARGET_OP, "kernels": KERNELS_PER_OP[TARGET_OP],
            "workload": "N=8 x fp32[16,777,216] (64 MiB per rank)",
            "us": t["us"], "achieved": t["GB/s"], "peak": peak, "unit": "GB/s",
            "frac": t["frac"], "frac_nominal": t["frac_nominal"],
            "algorithmic_bytes": bytes_[TARGET_OP], "traffic": recorded_traffic(TARGET_OP, count),
            "goal": ">= 0.70 of the HBM roofline for the fused FP8 allreduce on >= 16 MB messages"}
    if world == 1 and not args.only and not args.no_latency:
        res["small_messages"] = small_message_latency(dev)
    if world == 1 and not args.only and not args.no_workloads:
        del ops, step
        torch.cuda.empty_cache()
        res["workloads"] = workload_suite(dev, peak)
    if count != COUNT or args.only:
        res["config"]["workload"] = "PROFILING CASE, not the benchmark: %s on N=8 x fp32[%d]" % (
            ",".join(bytes_), count)
    if world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(x_host, sample=min(CPU_SAMPLE, count))
    return res


# ------------------------------------------------------------ small messages

def small_message_latency(dev, reps: int = 200, graph_reps: int = 50) -> dict:
    """Microseconds per call for the small-message workloads (decode-sized
    bf16 [32, 8192] x 8 ranks, and the [10, 20] fp32 quick-start shape), L2
    hot: back-to-back calls timed with CUDA events, once launched one by one
    from Python through the C ABI and once replayed from a CUDA graph (no
    host launch cost)."""
    import torch
    from precision_collective_reduction_fp32_b200 import binding as B
    from precision_collective_reduction_fp32_b200 import synth
    res = {}
    cases = [("decode_bf16_8x32x8192", 2, torch.bfloat16, B.RLX_BF16),
             ("tiny_fp32_8x10x20", 1, torch.float32, B.RLX_F32)]
    for name, wl, tdt, dcode in cases:
        xh = synth.rank_buffers(wl)
        x = torch.from_numpy(xh.view(np.int16) if tdt == torch.bfloat16 else xh).to(dev)
        x = x.view(tdt) if tdt == torch.bfloat16 else x
        n, c = x.shape
        out = torch.empty_like(x)
        ws = torch.empty(max(B.rlx_workspace_bytes(B.RLX_COLL_ALLREDUCE_TREE, c, n, dcode,
                                                   B.RLX_WIRE_FP8_E4M3), 16),
                         dtype=torch.uint8, device=dev)
        # the one-launch tree: zeroed synchronisation words (each call leaves them zero)
        fws = torch.zeros(B.rlx_workspace_bytes(B.RLX_COLL_ALLREDUCE_TREE_FUSED, c, n, dcode,
                                                B.RLX_WIRE_FP8_E4M3), dtype=torch.uint8, device=dev)
        row = {}
        for algo in ("flat", "tree", "tree_fused"):
            for wname, wire in (("native", B.RLX_WIRE_NATIVE), ("fp8", B.RLX_WIRE_FP8_E4M3)):
                def call(stream_ptr):
                    if algo == "flat":
                        B.rlx_allreduce_flat(x.data_ptr(), out.data_ptr(), c, c, n, dcode, wire,
                                             B.RLX_SUM, stream_ptr)
                    elif algo == "tree":
                        B.rlx_allreduce_tree(x.data_ptr(), out.data_ptr(), c, c, n, dcode, wire,
                                             B.RLX_SUM, ws.data_ptr(), ws.numel(), stream_ptr)
                    else:
                        B.rlx_allreduce_tree_fused(x.data_ptr(), out.data_ptr(), c, c, n, dcode,
                                                   wire, B.RLX_SUM, fws.data_ptr(), fws.numel(),
                                                   None, 0, stream_ptr)
                st = torch.cuda.current_stream(dev)
                for _ in range(20):
                    call(st.cuda_stream or None)
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(st)
                for _ in range(reps):
                    call(st.cuda_stream or None)
                e1.record(st)
                torch.cuda.synchronize()
                direct = e0.elapsed_time(e1) / reps * 1e3
                g = torch.cuda.CUDAGraph()
                cs = torch.cuda.Stream(dev)
                with torch.cuda.stream(cs):
                    call(cs.cuda_stream)
                    torch.cuda.synchronize()
                    with torch.cuda.graph(g, stream=cs):
                        for _ in range(graph_reps):
                            call(cs.cuda_stream)
                g.replay()
                torch.cuda.synchronize()
                e0.record(st)
                for _ in range(5):
                    g.replay()
                e1.record(st)
                torch.cuda.synchronize()
                graphed = e0.elapsed_time(e1) / (5 * graph_reps) * 1e3
                del g
                row["%s_%s" % (algo, wname)] = {"us_direct": round(direct, 2),
                                                "us_graph": round(graphed, 2)}
        res[name] = row
    return res


# ------------------------------------------------- the other workloads

def _timed_us(call, stream, reps: int, warmup: int = 3) -> float:
    """Mean microseconds per call of `reps` back-to-back calls (CUDA events
    at the two ends, on the launching stream)."""
    import torch
    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps * 1e3


def _cold_us(call, stream, flush, reps: int, dirty: bool = True) -> float:
    """Median microseconds of one call with the L2 flushed before it, outside
    the events: by writing a buffer larger than L2 (dirty: the call's misses
    also evict lines that must be written back) or by reading one (clean)."""
    import torch
    call()
    torch.cuda.synchronize()
    ts = []
    sink = torch.empty((), dtype=torch.int64, device=flush.device)
    for _ in range(reps):
        if dirty:
            flush.zero_()
        else:
            torch.sum(flush, dim=0, dtype=torch.int64, out=sink)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call()
        e1.record(stream)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) * 1e3)
    return statistics.median(ts)


def workload_suite(dev, peak: float, reps: int = 20, scale: int = 1) -> dict:
    """Per-operation figures on the other full-size workloads, drawn on the
    device (same recipes as the host draws): decode bf16 [32, 8192] x 8 with
    the L2 cold (flushed by a write, and by a read), prefill bf16 [4096, 8192]
    x 8 (DDA-tree and -flat, reduce-scatter, all-gather, alltoall, both wires)
    and lp-collectives fp32 [67,108,864] x 8 (quantise, reduce-scatter,
    all-gather, alltoall, both wires)."""
    import torch
    from precision_collective_reduction_fp32_b200 import binding as B
    from precision_collective_reduction_fp32_b200 import synth
    st = torch.cuda.current_stream(dev)
    sp = st.cuda_stream or None
    NAT, FP8, SUM = B.RLX_WIRE_NATIVE, B.RLX_WIRE_FP8_E4M3, B.RLX_SUM
    wires = (("native", NAT), ("fp8", FP8))
    res = {}
    # scale > 1 divides every workload's count (profiling cases only)
    draw = lambda k: synth.device_rank_buffers(k, dev, count=synth.WORKLOADS[k].count // scale)

    def entry(us, nbytes):
        gbs = nbytes / (us * 1e-6) / 1e9
        return {"us": round(us, 2), "GB/s": round(gbs, 1), "frac": round(gbs / peak, 3),
                "MiB": round(nbytes / MIB, 2), "floor_us": round(nbytes / (peak * 1e9) * 1e6, 2)}

    def allreduces(x, dcode, esize, cold=None, dirty=True):
        n, c = x.shape
        out = torch.empty_like(x)
        ws = torch.empty(max(B.rlx_workspace_bytes(B.RLX_COLL_ALLREDUCE_TREE, c, n, dcode, FP8), 16),
                         dtype=torch.uint8, device=dev)
        fws = torch.zeros(B.rlx_workspace_bytes(B.RLX_COLL_ALLREDUCE_TREE_FUSED, c, n, dcode, FP8),
                          dtype=torch.uint8, device=dev)
        ob = op_bytes(c, n, esize)
        row = {}
        for algo in ("flat", "tree", "tree_fused"):
            for wname, wire in wires:
                if algo == "flat":
                    f = lambda w=wire: B.rlx_allreduce_flat(x.data_ptr(), out.data_ptr(), c, c, n,
                                                            dcode, w, SUM, sp)
                elif algo == "tree":
                    f = lambda w=wire: B.rlx_allreduce_tree(x.data_ptr(), out.data_ptr(), c, c, n,
                                                            dcode, w, SUM, ws.data_ptr(),
                                                            ws.numel(), sp)
                else:
                    f = lambda w=wire: B.rlx_allreduce_tree_fused(x.data_ptr(), out.data_ptr(), c, c,
                                                                  n, dcode, w, SUM, fws.data_ptr(),
                                                                  fws.numel(), None, 0, sp)
                # the one-launch tree moves the same algorithmic bytes as the tree
                nb = ob["allreduce_%s_%s" % ("tree" if algo == "tree_fused" else algo, wname)]
                us = _cold_us(f, st, cold, reps, dirty) if cold is not None else _timed_us(f, st, reps)
                row["allreduce_%s_%s" % (algo, wname)] = entry(us, nb)
        del out, ws, fws
        return row

    def chunked(x, dcode, esize, quantise):
        """quantise (optional), reduce-scatter, all-gather of its result and
        alltoall of x, both wires, on [N, c] rank buffers x."""
        n, c = x.shape
        m = c // n
        ob = op_bytes(c, n, esize)
        y = torch.empty_like(x)
        rs = torch.empty((n, m), dtype=x.dtype, device=dev)
        row = {}
        if quantise:
            codes = torch.empty((n, c), dtype=torch.uint8, device=dev)
            scales = torch.empty((n, (c + BLOCK - 1) // BLOCK), dtype=torch.float32, device=dev)
            row["quantize_fp8"] = entry(_timed_us(lambda: B.rlx_quantize_fp8(
                x.data_ptr(), dcode, n, c, c, codes.data_ptr(), scales.data_ptr(), sp), st, reps),
                ob["quantize_fp8"])
            del codes, scales
        for wname, wire in wires:
            row["reduce_scatter_" + wname] = entry(_timed_us(lambda: B.rlx_reduce_scatter(
                x.data_ptr(), c, rs.data_ptr(), m, m, n, dcode, wire, SUM, sp), st, reps),
                ob["reduce_scatter_" + wname])
            row["all_gather_" + wname] = entry(_timed_us(lambda: B.rlx_all_gather(
                rs.data_ptr(), m, y.data_ptr(), c, m, n, dcode, wire, sp), st, reps),
                ob["all_gather_" + wname])
            row["alltoall_" + wname] = entry(_timed_us(lambda: B.rlx_alltoall(
                x.data_ptr(), c, y.data_ptr(), c, m, n, dcode, wire, sp), st, reps),
                ob["alltoall_" + wname])
        return row

    # decode, L2 cold (the hot-L2 figures are under small_messages)
    flush = torch.empty(256 * MIB, dtype=torch.uint8, device=dev)
    x = draw(2)
    res["decode_bf16_8x32x8192_cold_l2"] = allreduces(x, B.RLX_BF16, 2, cold=flush)
    res["decode_bf16_8x32x8192_cold_l2_clean"] = allreduces(x, B.RLX_BF16, 2, cold=flush,
                                                           dirty=False)
    del x, flush
    # prefill, and the chunked collectives on the same bf16 rank buffers
    x = draw(3)
    res["prefill_bf16_8x4096x8192"] = allreduces(x, B.RLX_BF16, 2)
    res["prefill_bf16_8x4096x8192"].update(chunked(x, B.RLX_BF16, 2, quantise=False))
    del x
    # lp-collectives
    x = draw(5)
    res["lp_collectives_fp32_8x67108864"] = chunked(x, B.RLX_F32, 4, quantise=True)
    del x
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------- quotient ablation

def quotient_ablation(dev, reps: int = 20) -> dict:
    """Profiling mode: what the correctly rounded quotient costs.  Times the
    FP8-wire operations with the product build (quotient fl32(x / s) by
    Markstein corrections) and with the profiling builds of the same sources
    (build.VARIANTS: x * fl32(448 / amax); CUDA's IEEE division for every
    element; the codes from two bracketing products with the full quotient
    only where they disagree), on workload 4 (N=8 x fp32[16,777,216]) and on the bf16 prefill
    buffers (N=8 x bf16[33,554,432]), inputs drawn on the device; and counts
    the quantised codes and DDA-tree results in which each variant differs
    from the product build."""
    import torch
    from precision_collective_reduction_fp32_b200 import binding as B
    from precision_collective_reduction_fp32_b200 import build as rlx_build
    from precision_collective_reduction_fp32_b200 import synth
    libs = {"correctly_rounded (product)": B.lib()}
    for name in rlx_build.VARIANTS:
        libs[name] = B.load(rlx_build.build_variant(name))
    st = torch.cuda.current_stream(dev)
    sp = st.cuda_stream or None
    FP8, SUM = B.RLX_WIRE_FP8_E4M3, B.RLX_SUM

    def ok(rc):
        if rc != B.RLX_OK:
            raise RuntimeError("rlx call failed: %d" % rc)

    res = {"us": {}, "differs_from_product": {}}
    for wl, dcode, esize, tag in ((4, B.RLX_F32, 4, "lp_allreduce_fp32_8x16777216"),
                                  (3, B.RLX_BF16, 2, "prefill_bf16_8x33554432")):
        x = synth.device_rank_buffers(wl, dev)
        n, c = x.shape
        m = c // n
        y = torch.empty_like(x)
        rs = torch.empty((n, m), dtype=x.dtype, device=dev)
        codes = torch.empty((n, c), dtype=torch.uint8, device=dev)
        scales = torch.empty((n, c // BLOCK), dtype=torch.float32, device=dev)
        wsb = B.rlx_workspace_bytes(B.RLX_COLL_ALLREDUCE_TREE, c, n, dcode, FP8)
        ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
        ob = op_bytes(c, n, esize)
        ref_codes = ref_tree = None
        for lname, L in libs.items():
            calls = {
                "quantize_fp8": lambda: ok(L.rlx_quantize_fp8(x.data_ptr(), dcode, n, c, c,
                                                              codes.data_ptr(), scales.data_ptr(), sp)),
                "allreduce_flat_fp8": lambda: ok(L.rlx_allreduce_flat(x.data_ptr(), y.data_ptr(), c, c,
                                                                      n, dcode, FP8, SUM, sp)),
                "allreduce_tree_fp8": lambda: ok(L.rlx_allreduce_tree(x.data_ptr(), y.data_ptr(), c, c,
                                                                      n, dcode, FP8, SUM, ws.data_ptr(),
                                                                      wsb, sp)),
                "reduce_scatter_fp8": lambda: ok(L.rlx_reduce_scatter(x.data_ptr(), c, rs.data_ptr(), m,
                                                                      m, n, dcode, FP8, SUM, sp)),
                "all_gather_fp8": lambda: ok(L.rlx_all_gather(rs.data_ptr(), m, y.data_ptr(), c, m, n,
                                                              dcode, FP8, sp)),
                "alltoall_fp8": lambda: ok(L.rlx_alltoall(x.data_ptr(), c, y.data_ptr(), c, m, n,
                                                          dcode, FP8, sp)),
            }
            row = {}
            for op, f in calls.items():
                us = _timed_us(f, st, reps)
                row[op] = {"us": round(us, 2), "GB/s": round(ob[op] / (us * 1e-6) / 1e9, 1)}
            row["fp8_ops_total_us"] = round(sum(v["us"] for v in row.values()), 1)
            res["us"].setdefault(lname, {})[tag] = row
            calls["quantize_fp8"]()
            calls["allreduce_tree_fp8"]()
            torch.cuda.synchronize()
            if ref_codes is None:
                ref_codes, ref_tree = codes.clone(), y.clone()
            else:
                it = torch.int16 if x.dtype == torch.bfloat16 else torch.int32
                res["differs_from_product"].setdefault(lname, {})[tag] = {
                    "quantize_codes": int((codes != ref_codes).sum().item()),
                    "codes_total": codes.numel(),
                    "tree_fp8_elements": int((y.view(it) != ref_tree.view(it)).sum().item()),
                    "elements_total": y.numel()}
        del x, y, rs, codes, scales, ws, ref_codes, ref_tree
        torch.cuda.empty_cache()
    return res


# --------------------------------------------------------------- CPU oracle

def oracle_step(xs: np.ndarray) -> None:
    """The same twelve operations, run by the CPU oracle on a sample."""
    import oracle
    n, c = xs.shape
    m = c // n
    codes, scales = oracle.quantize(xs)
    oracle.dequantize(codes, scales)
    for w in (oracle.NATIVE, oracle.FP8):
        oracle.allreduce_flat(xs, wire=w)
        oracle.allreduce_tree(xs, wire=w)
        rs = oracle.reduce_scatter(xs, m, wire=w)
        oracle.all_gather(rs, m, wire=w)
        oracle.alltoall(xs, m, wire=w)


def cpu_baseline(x_host: np.ndarray, sample: int = CPU_SAMPLE, repeats: int = 1) -> dict:
    import oracle
    oracle.build()
    xs = np.ascontiguousarray(x_host[:, :sample])
    t0 = time.perf_counter()
    for _ in range(repeats):
        oracle_step(xs)
    dt = time.perf_counter() - t0
    b = sum(op_bytes(sample, NRANKS).values()) * repeats
    return {"value": round(b / dt / 1e9, 3), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "host_cores": os.cpu_count(),
            "sample": "%d pass(es) of the twelve operations on the first %d elements of each of "
                      "the %d ranks (1/%d of the batch), single-threaded C oracle; %.1f s"
                      % (repeats, sample, NRANKS, COUNT // sample, dt)}


def run_reference(args, rank: int) -> dict | None:
    """The reference arm: the CPU oracle as it stands, on bounded samples."""
    if rank != 0:
        return None
    from precision_collective_reduction_fp32_b200 import synth
    sample = args.ref_sample
    xs = np.empty((NRANKS, sample), dtype=np.float32)
    for r in range(NRANKS):
        xs[r] = synth.draw_row("normal_outliers", sample, synth.seed(WORKLOAD, r))
    for _ in range(args.warmup):
        oracle_step(xs)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(xs)
    dt = time.perf_counter() - t0
    b = sum(op_bytes(sample, NRANKS).values()) * args.steps
    value = b / dt / 1e9
    desc = ("each step: the twelve operations on the first %d elements of each of the %d ranks "
            "(1/%d of the batch), single-threaded C oracle" % (sample, NRANKS, COUNT // sample))
    return {"impl": "reference",
            "metric": "emulated N=8 allreduce effective HBM GB/s (fp32 & FP8) and % of B200 HBM peak",
            "value": round(value, 3), "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": "N=8 simulated ranks x fp32[16,777,216], N(0,1) with 1% x100 "
                                   "outliers (bounded sample, see cpu_baseline)",
                       "nranks": NRANKS, "count": COUNT},
            "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": 1,
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["rlx", "reference"], default="rlx")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--ref-sample", type=int, default=262_144)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-latency", action="store_true",
                    help="skip the small-message latency figures")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the per-operation figures on the other workloads")
    ap.add_argument("--suite-only", action="store_true",
                    help="profiling: run only the other workloads' per-operation figures "
                         "(--steps calls each)")
    ap.add_argument("--suite-scale", type=int, default=1,
                    help="profiling: divide the other workloads' counts by this")
    ap.add_argument("--quotient-ablation", action="store_true",
                    help="profiling: time the FP8 operations with the correctly rounded "
                         "quotient against three profiling builds (reciprocal multiply, IEEE "
                         "division for every element, bracketing products); --steps calls each")
    ap.add_argument("--count", type=int, default=COUNT,
                    help="elements per rank (profiling cases only; the benchmark is 16,777,216)")
    ap.add_argument("--only", default="",
                    help="comma-separated operations to run (profiling cases only)")
    args = ap.parse_args(argv)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.suite_only:
        # profiling case: the per-operation figures of the other workloads
        # only, every count divided by --suite-scale
        import torch
        torch.cuda.set_device(0)
        print(json.dumps({"workloads": workload_suite(torch.device("cuda", 0), peaks()[0],
                                                      reps=args.steps, scale=args.suite_scale),
                          "note": "PROFILING CASE, counts / %d" % args.suite_scale}), flush=True)
        return 0
    if args.quotient_ablation:
        import torch
        torch.cuda.set_device(0)
        print(json.dumps({"quotient_ablation": quotient_ablation(torch.device("cuda", 0),
                                                                 reps=args.steps),
                          "note": "PROFILING CASE: product build against profiling builds"}),
              flush=True)
        return 0
    if args.impl == "reference":
        res = run_reference(args, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        res = run_gpu(args, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if res is not None:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
