"""The benchmark's end-to-end leg (bench.E2ETreeFp8) cuts each step into
column ranges and reduces each with its own rlx_allreduce_tree call on the
strided rows.  Its host output must be the DDA-tree result of the whole rows,
bit for bit: every 128-block lies inside one range, and the tree's result
does not depend on its chunking.  Checked against the oracle for several
steps (both device batches), with ranges and without (a count that is no
multiple of the block size runs as one range)."""
import numpy as np
import pytest
import torch

import bench
import oracle
import refpipe
from precision_collective_reduction_fp32_b200 import build as rlx_build
from precision_collective_reduction_fp32_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    rlx_build.build()
    oracle.build()


@pytest.mark.parametrize("count,slices,expect", [(128 * 6 * 8, 8, 8), (128 * 9 * 4, 8, 6),
                                                 (1000, 8, 1)])
def test_e2e_ranges_match_oracle(count, slices, expect):
    x = np.stack([synth.draw_row("normal_outliers", count, 900 + r) for r in range(8)])
    e = bench.E2ETreeFp8(x, torch.device("cuda", 0), slices=slices)
    assert e.slices == expect
    ref = oracle.allreduce_tree(x, wire=oracle.FP8)
    ms = e(3)
    assert ms > 0
    for k in (1, 2):
        assert refpipe.same_bits(e.result(k).numpy(), ref), "step %d" % k
