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


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _deps())


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
          lib: str = LIB, obj: str = OBJ) -> str:
    if not force and not stale(lib):
        return lib
    os.makedirs(obj, exist_ok=True)
    flags = FLAGS + list(extra or [])

    def compile_one(src: str) -> str:
        o = os.path.join(obj, os.path.basename(src)[:-3] + ".o")
        cmd = [NVCC, *flags, "-c", src, "-o", o]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc failed for %s:\n%s%s" % (src, r.stdout, r.stderr))
        if verbose and (r.stdout or r.stderr):
            sys.stderr.write(r.stdout + r.stderr)
        return o

    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, sources()))

    vmap = os.path.join(obj, "rlx.map")
    with open(vmap, "w") as f:
        f.write("{ global: rlx_*; local: *; };\n")
    os.makedirs(os.path.dirname(lib), exist_ok=True)
    tmp = lib + ".tmp.%d" % os.getpid()
    cmd = [NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-Xlinker", "--version-script=" + vmap]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("link failed:\n%s%s" % (r.stdout, r.stderr))
    os.replace(tmp, lib)
    return lib


# Profiling builds: the same sources with one compile-time switch changed,
# written under _build/variants/<name>/ (never next to the package, so the
# package always loads the product build).  Used by bench.py's ablation mode.
VARIANTS = {
    # quotient x * fl32(448 / amax) instead of the correctly rounded x / s
    "recip_quotient": ["-DRLX_QUOTIENT=1"],
    # CUDA's IEEE division for every element
    "ieee_div_quotient": ["-DRLX_QUOTIENT=2"],
    # the correctly rounded quotient's codes from two bracketing products,
    # the full quotient only where the bracket is not decisive
    "bracket_quotient": ["-DRLX_QUOTIENT=3"],
}


def build_variant(name: str, force: bool = False) -> str:
    base = os.path.join(ROOT, "_build", "variants", name)
    return build(force=force, extra=VARIANTS[name], lib=os.path.join(base, "librlx.so"),
                 obj=os.path.join(base, "obj"))


if __name__ == "__main__":
    force = "--force" in sys.argv
    verbose = "-v" in sys.argv
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None
    print(build(force=force, verbose=verbose or bool(extra), extra=extra))
