"""The work plan of the one-launch DDA-tree, on the CPU: a host-only program
built from the kernel's own plan functions (rlx_tree_plan.cuh) checks, for
476 shapes (17 counts x 7 rank counts x 2 dtypes x 2 wires), that the ticket
order is a bijection onto the runs, that every all-gather run is handed out
after all the reduce-scatter work of the chunks it reads (what the kernel's
no-deadlock argument rests on), and that each chunk's ready target equals
the work that reports to it."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def test_tree_plan_order_and_targets(tmp_path):
    exe = str(tmp_path / "tree_plan_check")
    subprocess.check_call(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-std=c++20", "-O2", "-o", exe,
                           os.path.join(HERE, "cuda", "tree_plan_check.cu")])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "ok: 476 shapes" in r.stdout
