"""The kernels split a unit index into (segment, offset) with a multiply-shift
divider (Granlund & Montgomery 1994).  This builds a host-only program from
the library's device header and compares it with integer division (CPU)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def test_fastdiv_matches_integer_division(tmp_path):
    exe = str(tmp_path / "fastdiv_check")
    subprocess.check_call(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-std=c++20", "-O2", "-o", exe,
                           os.path.join(HERE, "cuda", "fastdiv_check.cu")])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
