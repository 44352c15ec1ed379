"""The job-wide low-precision switch (the pages' RCCL_LOW_PRECISION_ENABLE=1):
with wire=None the Python helpers take the FP8 wire when the variable is "1"
and the native wire otherwise; an explicit wire always wins (CPU only)."""
import pytest

import precision_collective_reduction_fp32_b200 as rlx
from precision_collective_reduction_fp32_b200 import binding as B


@pytest.mark.parametrize("var", rlx.LOW_PRECISION_ENV)
def test_env_switch(monkeypatch, var):
    for v in rlx.LOW_PRECISION_ENV:
        monkeypatch.delenv(v, raising=False)
    assert rlx.default_wire() == "native" and rlx._wire(None) == B.RLX_WIRE_NATIVE
    monkeypatch.setenv(var, "1")
    assert rlx.default_wire() == "fp8" and rlx._wire(None) == B.RLX_WIRE_FP8_E4M3
    assert rlx._wire("native") == B.RLX_WIRE_NATIVE
    monkeypatch.setenv(var, "0")
    assert rlx.default_wire() == "native"


def test_bad_wire_rejected():
    with pytest.raises(ValueError):
        rlx._wire("fp4")
