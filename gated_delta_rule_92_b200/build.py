"""Build the sm_100a CUDA libraries in-tree (nvcc, no JIT): ``libgdn2.so`` and
its debug build ``libgdn2_debug.so`` (the same sources with -DGDN2_DEBUG_BOUNDS:
device-side range checks that record a status instead of trapping)."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "gdn2_lib.cu")
# the no-alloc host entry keeps its device array in a translation unit of its own
SRC_NOALLOC = os.path.join(HERE, "csrc", "gdn2_noalloc.cu")
LIB = os.path.join(HERE, "libgdn2.so")
DEBUG_LIB = os.path.join(HERE, "libgdn2_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
]
DEBUG_FLAGS = ["-DGDN2_DEBUG_BOUNDS"]


def _sources():
    return [SRC, SRC_NOALLOC] + glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + \
        [os.path.join(os.path.dirname(HERE), "include", "gdn2.h")]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(s) <= t for s in _sources())


def _cmd(lib: str, extra, verbose: bool):
    return [NVCC] + FLAGS + list(extra) + (["-Xptxas", "-v"] if verbose else []) + \
        ["-o", lib, SRC, SRC_NOALLOC, "-ldl", "-lpthread", "-lrt"]


def build(force: bool = False, verbose: bool = False, debug: bool = True) -> str:
    """Compile the release library (and, with `debug`, the debug build beside
    it; the two nvcc runs go in parallel).  Returns the release library's path."""
    jobs = [(LIB, [])] + ([(DEBUG_LIB, DEBUG_FLAGS)] if debug else [])
    procs = [subprocess.Popen(_cmd(lib, extra, verbose)) for lib, extra in jobs
             if force or not up_to_date(lib)]
    failed = [p.args for p in procs if p.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, failed[0])
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--no-debug" not in sys.argv)
    print(LIB)
