"""Build libw4a16.so (sm_100a) in-tree with nvcc.

    python -m w4a16_matmul_pack_b200.build [--verbose]
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC_DIR = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libw4a16.so")
MAIN = os.path.join(SRC_DIR, "w4a16.cu")
UNITS = [MAIN, os.path.join(SRC_DIR, "noalloc.cu")]

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
    "--expt-relaxed-constexpr",
    # IEEE binary32 division/sqrt and no flush-to-zero: the packer must take the
    # same rounding decisions as the specification.
    "-prec-div=true", "-prec-sqrt=true", "-ftz=false", "-fmad=true",
]


def _sources():
    return [os.path.join(SRC_DIR, f) for f in sorted(os.listdir(SRC_DIR))
            if f.endswith((".cu", ".cuh"))] + [os.path.join(HERE, "..", "include", "w4a16.h")]


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = LIB + f".{os.getpid()}.tmp"
    cmd = [nvcc, *NVCC_FLAGS, *UNITS, "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
