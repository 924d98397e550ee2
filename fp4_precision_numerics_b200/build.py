"""Build libmxfp4.so in-tree: one nvcc translation unit for sm_100a.

    python -m fp4_precision_numerics_b200.build [--verbose]

Flags: -gencode arch=compute_100a,code=sm_100a, -O3, -lineinfo; no
--use_fast_math (binary32 rounding and subnormals are part of the bit
contract).  The shared object lands next to this file and travels with the
source tree; nothing is installed elsewhere.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC_DIR = os.path.join(HERE, "csrc")
SOURCES = [os.path.join(SRC_DIR, "mxfp4_api.cu")]
DEPS = [os.path.join(SRC_DIR, f) for f in os.listdir(SRC_DIR) if f.endswith((".cu", ".cuh"))] + [
    os.path.join(ROOT, "include", "mxfp4.h")]
LIB = os.path.join(HERE, "libmxfp4.so")

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-shared",
              "-I" + os.path.join(ROOT, "include"), "-lcudart"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = [nvcc()] + NVCC_FLAGS + (["-Xptxas", "-v"] if verbose else []) + ["-o", tmp] + SOURCES
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
