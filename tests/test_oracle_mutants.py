"""The oracle's pins catch plausible mistakes (CPU only).

Each mutant is oracle.c with one small, plausible slip planted in a temporary
copy (a dropped rank, a reciprocal instead of a division, ties rounded away
from zero, a transposed alltoall index, ...).  The pin tests are run against
the mutant's build; at least one of them must fail.  The committed oracle is
never modified.
"""
import os
import shutil
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(ROOT, "oracle", "oracle.c")

# (name, original text, replacement) -- each original must occur exactly once.
MUTANTS = [
    ("drop_last_rank", "for (int s = 0; s < nranks; ++s) {\n        load_f32(dtype, send, stride, (size_t)s, off",
     "for (int s = 0; s < nranks - 1; ++s) {\n        load_f32(dtype, send, stride, (size_t)s, off"),
    ("reciprocal_scale", "orc_e4m3_encode(x[i] / s)", "orc_e4m3_encode(x[i] * (1.0f / s))"),
    ("ties_away", "if (rem > half || (rem == half && (q & 1u)))", "if (rem >= half)"),
    ("saturate_at_480", "if (a >= 0x43E00000u)", "if (a >= 0x43F00000u)"),
    ("alltoall_transposed", "copy_elems(dtype, send, send_stride, (size_t)s, (size_t)r * m,\n"
     "                           recv, recv_stride, (size_t)r, (size_t)s * m, m);",
     "copy_elems(dtype, send, send_stride, (size_t)s, (size_t)s * m,\n"
     "                           recv, recv_stride, (size_t)r, (size_t)r * m, m);"),
    ("tree_chunk_floor", "size_t per_rank = (blocks + (size_t)nranks - 1) / (size_t)nranks;",
     "size_t per_rank = blocks / (size_t)nranks + 1;"),
    ("amax_skips_last", "for (size_t i = 0; i < len; ++i) {\n        float ax = fabsf(x[i]);",
     "for (size_t i = 0; i + 1 < len; ++i) {\n        float ax = fabsf(x[i]);"),
    ("bf16_truncates", "u += 0x7FFFu + lsb;", "u += 0x8000u;"),
    ("dequant_first_scale", "dequant_block(codes + lo, n, scales[b], y + lo);",
     "dequant_block(codes + lo, n, scales[0], y + lo);"),
    ("zero_block_drops_sign", "codes[i] = signbit(x[i]) ? 0x80 : 0x00;", "codes[i] = 0x00;"),
    ("tree_skips_requant", "dequant_segment(pay_codes + lo, pay_scales + lo / ORC_BLOCK, len, chunk);",
     "reduce_segment(dtype, 1, send, stride, lo, len, nranks, chunk);"),
    ("subnormal_shift_off_by_one", "return sign | (uint8_t)round_shift_rne(sig, -(pow2 + 9));",
     "return sign | (uint8_t)round_shift_rne(sig, -(pow2 + 8));"),
    ("sum_from_zero_drops_sign", "            for (size_t i = 0; i < len; ++i)\n                sum[i] = term[i];",
     "            for (size_t i = 0; i < len; ++i)\n                sum[i] = 0.0f + term[i];"),
]

PIN_TESTS = [
    os.path.join(HERE, "test_oracle_codec.py") + "::test_encode_ties_and_neighbours_bruteforce",
    os.path.join(HERE, "test_oracle_codec.py") + "::test_encode_random_bruteforce",
    os.path.join(HERE, "test_oracle_codec.py") + "::test_bf16_rne_vs_torch",
    os.path.join(HERE, "test_oracle_collectives.py"),
]


def _build_mutant(tmp, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, name
    d = os.path.join(tmp, name)
    os.makedirs(d)
    shutil.copy(os.path.join(ROOT, "oracle", "oracle.h"), d)
    with open(os.path.join(d, "oracle.c"), "w") as f:
        f.write(src.replace(old, new))
    so = os.path.join(d, "liboracle.so")
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fPIC", "-shared", "-std=c99",
                           "-o", so, os.path.join(d, "oracle.c"), "-lm"])
    return so


def _run_pins(so):
    env = dict(os.environ, ORACLE_LIB=so)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        *PIN_TESTS], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode


def test_every_mutant_is_caught():
    # The first entry is an unmodified copy: the harness itself must pass it,
    # otherwise every "caught" mutant would prove nothing.
    control = ("control", "#define ORC_BLOCK 128", "#define ORC_BLOCK 128")
    with tempfile.TemporaryDirectory() as tmp:
        libs = [(name, _build_mutant(tmp, name, old, new))
                for name, old, new in [control] + MUTANTS]
        with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            rcs = dict(ex.map(lambda nl: (nl[0], _run_pins(nl[1])), libs))
    assert rcs.pop("control") == 0, "the unmodified oracle failed its own pins"
    survivors = [name for name, rc in rcs.items() if rc == 0]
    assert not survivors, "pins did not catch: %s" % survivors
