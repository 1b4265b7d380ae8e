"""Build libssm.so (the CUDA library behind include/ssm.h) in-tree for sm_100a.

Usage: ``python -m selective_state_space_45_b200.build [--verbose]``.  nvcc cross-compiles
without a GPU; the .so lands next to this file and is what the Python binding loads.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libssm.so")
SOURCES = [os.path.join(CSRC, "ssm_api.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("common.cuh", "conv1d.cuh", "scan_fwd.cuh", "state_step.cuh")] + [
    os.path.join(ROOT, "include", "ssm.h")]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2", "-shared",
    "-I", os.path.join(ROOT, "include"),
]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = [NVCC] + FLAGS + (["-Xptxas", "-v"] if verbose else []) + SOURCES + ["-o", tmp]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
