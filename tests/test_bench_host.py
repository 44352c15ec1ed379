"""Host-side logic of bench.py, on CPU: the algorithmic byte model against
the totals worked out by hand for the benchmark workloads, the launch count,
the reference arm's JSON line (the oracle on a tiny sample), and the rule
that a recorded DRAM traffic figure is used only for the kernels it was
measured on."""
import json

import pytest

import bench

MIB = 1 << 20


def test_op_bytes_lp_allreduce_totals():
    """N=8 x fp32[16,777,216]: inputs read once, outputs written once, the
    DDA-tree FP8 payload (codes + one fp32 scale per 128-block) written and
    read once; flat's N^2 interconnect reads are not HBM bytes."""
    b = bench.op_bytes(16_777_216, 8)
    want = {"quantize_fp8": 644, "dequantize_fp8": 644, "allreduce_flat_native": 1024,
            "allreduce_flat_fp8": 1024, "allreduce_tree_native": 1088,
            "allreduce_tree_fp8": 1057, "reduce_scatter_native": 576,
            "reduce_scatter_fp8": 576, "all_gather_native": 576, "all_gather_fp8": 576,
            "alltoall_native": 1024, "alltoall_fp8": 1024}
    assert {k: v / MIB for k, v in b.items()} == want
    assert sum(b.values()) == 9833 * MIB          # 9.6 GiB per step


def test_op_bytes_other_workloads():
    # prefill, bf16 [4096, 8192] x 8: DDA-tree native = 17 rank buffers of 64 MiB
    assert bench.op_bytes(4096 * 8192, 8, esize=2)["allreduce_tree_native"] == 17 * 64 * MIB
    # lp-collectives, fp32 [67,108,864] x 8
    b = bench.op_bytes(67_108_864, 8)
    assert b["reduce_scatter_fp8"] == 2304 * MIB          # 2 GiB in, 256 MiB out
    assert b["all_gather_fp8"] == 2304 * MIB
    assert b["alltoall_fp8"] == 4096 * MIB
    assert b["quantize_fp8"] == 2048 * MIB + 512 * MIB + 16 * MIB


def test_launch_count_per_step():
    assert sum(bench.KERNELS_PER_OP.values()) == 14
    assert bench.KERNELS_PER_OP["allreduce_tree_fp8"] == 2
    assert bench.KERNELS_PER_OP["allreduce_flat_fp8"] == 1


def test_reference_arm_json(capsys):
    args = bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0",
                       "--ref-sample", "1024"])
    assert args == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"):
        assert k in line
    assert line["value"] > 0 and line["unit"] == "GB/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_recorded_traffic_needs_matching_kernels(monkeypatch):
    real = bench.source_hash()
    rec = bench.recorded_traffic("allreduce_flat_fp8")
    if rec is None:
        pytest.skip("no traffic record for the current kernel sources")
    assert 0.9 * 1024 * MIB < rec <= 1024 * MIB
    # a record taken at another size does not describe this launch
    assert bench.recorded_traffic("allreduce_flat_fp8", bench.COUNT // 4) is None
    monkeypatch.setattr(bench, "source_hash", lambda: real[::-1])
    assert bench.recorded_traffic("allreduce_flat_fp8") is None


def test_peaks_reads_measured_or_falls_back():
    peak, kind = bench.peaks()
    assert kind in ("measured", "fallback")
    assert peak > 1000
