"""Build librlx.so (the CUDA library) in-tree for sm_100a.

    python -m precision_collective_reduction_fp32_b200.build [--force]

Compiles csrc/*.cu with nvcc in parallel (objects under _build/ at the repo
root) and links them into librlx.so next to this file, exporting only the
rlx_* entry points declared in include/rlx.h.  Floating-point flags keep every
operation IEEE round-to-nearest: no FMA contraction, correctly rounded
division, no flush-to-zero.
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OBJ = os.path.join(ROOT, "_build", "rlx")
LIB = os.path.join(PKG, "librlx.so")
HEADERS = [os.path.join(ROOT, "include", "rlx.h")]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++20", "-fmad=false", "-prec-div=true",
                "-prec-sqrt=true", "-ftz=false", "-Xcompiler", "-fPIC",
                "-Xcompiler", "-fvisibility=hidden", "-Xptxas", "-warn-spills"]


def sources() -> list[str]:
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _deps() -> list[str]:
    return sources() + HEADERS + [os.path.join(CSRC, f) for f in os.listdir(CSRC)
                                  if f.endswith((".cuh", ".h"))]


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in _deps())


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None) -> str:
    if not force and not stale():
        return LIB
    os.makedirs(OBJ, exist_ok=True)
    flags = FLAGS + list(extra or [])

    def compile_one(src: str) -> str:
        obj = os.path.join(OBJ, os.path.basename(src)[:-3] + ".o")
        cmd = [NVCC, *flags, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc failed for %s:\n%s%s" % (src, r.stdout, r.stderr))
        if verbose and (r.stdout or r.stderr):
            sys.stderr.write(r.stdout + r.stderr)
        return obj

    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, sources()))

    vmap = os.path.join(OBJ, "rlx.map")
    with open(vmap, "w") as f:
        f.write("{ global: rlx_*; local: *; };\n")
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = [NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-Xlinker", "--version-script=" + vmap]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("link failed:\n%s%s" % (r.stdout, r.stderr))
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    force = "--force" in sys.argv
    verbose = "-v" in sys.argv
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None
    print(build(force=force, verbose=verbose or bool(extra), extra=extra))
