"""The seeded input generators (no arithmetic of the collectives): the
workload table, determinism, and that the bench's device-side draw follows
the same recipe as the host draw (on the CPU device the two give the same
bytes)."""
import numpy as np
import torch

from precision_collective_reduction_fp32_b200 import synth


def test_workload_table():
    w = synth.WORKLOADS
    assert (w[1].nranks, w[1].count, w[1].dtype) == (8, 200, "f32")
    assert (w[2].count, w[2].dtype, w[2].std) == (32 * 8192, "bf16", 0.5)
    assert (w[3].count, w[3].dtype) == (4096 * 8192, "bf16")
    assert (w[4].count, w[4].dist) == (16_777_216, "normal_outliers")
    assert (w[5].count, w[5].dist) == (67_108_864, "student_t3")
    assert all(x.nranks == 8 for x in w.values())


def test_seeded_and_distinct():
    a = synth.rank_buffers(4, count=5000, nranks=3)
    b = synth.rank_buffers(4, count=5000, nranks=3)
    assert np.array_equal(a, b)
    assert not np.array_equal(a[0], a[1])                        # ranks differ
    assert not np.array_equal(a, synth.rank_buffers(5, count=5000, nranks=3))


def test_padding_marker():
    x = synth.rank_buffers(1, count=10, nranks=2, stride=16)
    assert np.all(x[:, 10:] == np.float32(-7.25))
    xb = synth.rank_buffers(2, count=10, nranks=2, stride=16)
    assert np.all(xb[:, 10:] == 0xC0E8)


def test_device_draw_is_the_host_recipe():
    for k, count in ((1, 200), (2, 4096), (4, 70_000), (5, 3000)):
        host = synth.rank_buffers(k, count=count)
        dev = synth.device_rank_buffers(k, "cpu", count=count)
        if synth.WORKLOADS[k].dtype == "bf16":
            got = dev.view(torch.int16).numpy().view(np.uint16)
        else:
            got = dev.numpy()
        assert np.array_equal(got, host), k


def test_outlier_and_tail_shapes():
    x = synth.rank_buffers(4, count=200_000, nranks=1)[0]
    big = np.abs(x) > 10
    assert 0.005 < big.mean() < 0.015                            # ~1 % scaled x100
    t = synth.rank_buffers(5, count=200_000, nranks=1)[0]
    assert np.abs(t).max() > 20 and 0.5 < np.median(np.abs(t)) < 1.0   # heavy tail, t(3)
