"""Build the sm_100a CUDA library ``libgdn2.so`` in-tree (nvcc, no JIT)."""
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
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
]


def _sources():
    return [SRC, SRC_NOALLOC] + glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + \
        [os.path.join(os.path.dirname(HERE), "include", "gdn2.h")]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(s) <= t for s in _sources())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    cmd = [NVCC] + FLAGS + (["-Xptxas", "-v"] if verbose else []) + \
        ["-o", LIB, SRC, SRC_NOALLOC, "-ldl", "-lpthread", "-lrt"]
    subprocess.check_call(cmd)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
