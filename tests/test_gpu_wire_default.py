"""The job-wide low-precision switch on the GPU.

The pages turn the FP8 collectives on for a whole job with an environment
variable ("Coletivos de Baixa Precisão — Compressão FP8 com Precisão FP32",
infolabhq summary: RCCL_LOW_PRECISION_ENABLE=1) and let users enable them
per call ("Colectivos de mengua precisión", RCCLX post, Spanish copy).  Here
the Python helpers called with wire=None take the FP8 wire when
RLX_LOW_PRECISION_ENABLE or RCCL_LOW_PRECISION_ENABLE is "1" and the native
wire otherwise; an explicit wire= always wins.  Every collective is run
through the helpers on the GPU and compared bit for bit with the oracle's
result for the wire the switch should have picked.
"""
import numpy as np
import pytest
import torch

import oracle
import precision_collective_reduction_fp32_b200 as rlx
from gpuutil import to_dev, to_host
from precision_collective_reduction_fp32_b200 import build as rlx_build
from precision_collective_reduction_fp32_b200 import synth

pytestmark = pytest.mark.gpu

N, M = 8, 3 * 128 + 40          # 8 ranks, chunks with a partial FP8 block
COUNT = N * M


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    rlx_build.build()
    oracle.build()


def _same(a, b):
    a, b = np.ascontiguousarray(a), np.ascontiguousarray(b)
    return a.shape == b.shape and np.array_equal(a.view(np.uint8), b.view(np.uint8))


def _run_all(x, wire):
    """Every collective through the Python helpers with the given wire
    argument (None: the job-wide default)."""
    dx = to_dev(x)
    out = {}
    for algo in ("flat", "tree"):
        out[algo] = rlx.allreduce(dx, algo=algo, wire=wire)
    rs = rlx.reduce_scatter(dx, wire=wire)
    out["reduce_scatter"] = rs
    out["all_gather"] = rlx.all_gather(rs, wire=wire)
    out["alltoall"] = rlx.alltoall(dx, wire=wire)
    torch.cuda.synchronize()
    return {k: to_host(v) for k, v in out.items()}


def _oracle_all(x, owire):
    rs = oracle.reduce_scatter(x, M, wire=owire)
    return {"flat": oracle.allreduce_flat(x, wire=owire),
            "tree": oracle.allreduce_tree(x, wire=owire),
            "reduce_scatter": rs,
            "all_gather": oracle.all_gather(rs, M, wire=owire),
            "alltoall": oracle.alltoall(x, M, wire=owire)}


def _clear(monkeypatch):
    for v in rlx.LOW_PRECISION_ENV:
        monkeypatch.delenv(v, raising=False)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("var", rlx.LOW_PRECISION_ENV)
def test_switch_on_selects_fp8(monkeypatch, var, dtype):
    x = synth.rank_buffers(4, count=COUNT, nranks=N, dtype=dtype)
    ref8, refn = _oracle_all(x, oracle.FP8), _oracle_all(x, oracle.NATIVE)
    _clear(monkeypatch)
    monkeypatch.setenv(var, "1")
    got = _run_all(x, None)
    for k in ref8:
        assert _same(got[k], ref8[k]), ("switch on, wire=None", k)
        assert not _same(got[k], refn[k]), ("FP8 result equals the native one", k)
    # an explicit wire wins over the switch
    got = _run_all(x, "native")
    for k in refn:
        assert _same(got[k], refn[k]), ("switch on, wire='native'", k)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_switch_off_selects_native(monkeypatch, dtype):
    x = synth.rank_buffers(5, count=COUNT, nranks=N, dtype=dtype)
    ref8, refn = _oracle_all(x, oracle.FP8), _oracle_all(x, oracle.NATIVE)
    _clear(monkeypatch)
    got = _run_all(x, None)
    for k in refn:
        assert _same(got[k], refn[k]), ("switch unset, wire=None", k)
    for v in rlx.LOW_PRECISION_ENV:
        monkeypatch.setenv(v, "0")
    got = _run_all(x, None)
    for k in refn:
        assert _same(got[k], refn[k]), ("switch '0', wire=None", k)
    # an explicit FP8 wire is honoured with the switch off
    got = _run_all(x, "fp8")
    for k in ref8:
        assert _same(got[k], ref8[k]), ("switch off, wire='fp8'", k)
