"""Build libssm.so (the CUDA library behind include/ssm.h) in-tree for sm_100a.

Usage: ``python -m selective_state_space_45_b200.build [--verbose]``.  nvcc cross-compiles
without a GPU.  Each translation unit of ``csrc/`` (one per operation of the C ABI) is
compiled to an object under ``_build/`` in parallel and only when it or a header it
includes changed; the objects are then linked into the .so next to this file, which is
what the Python binding loads.
"""
from __future__ import annotations

import concurrent.futures
import hashlib
import os
import re
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OBJDIR = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libssm.so")
UNITS = ["ssm_api.cu", "scan_api.cu", "step_api.cu", "conv_api.cu", "bwd_api.cu", "ssd_api.cu"]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
                 "-I", os.path.join(ROOT, "include")]

_INCLUDE = re.compile(r'^\s*#\s*include\s+"([^"]+)"', re.M)


def dependency_files(unit: str) -> list[str]:
    """The translation unit ``unit`` (a file name in csrc/) and every local header it
    includes, directly or not, as absolute paths in a stable order."""
    seen, order, todo = set(), [], [os.path.join(CSRC, unit)]
    while todo:
        path = os.path.normpath(todo.pop())
        if path in seen or not os.path.exists(path):
            continue
        seen.add(path)
        order.append(path)
        with open(path) as f:
            for inc in _INCLUDE.findall(f.read()):
                todo.append(os.path.join(os.path.dirname(path), inc))
    return sorted(order)


def source_hash(unit: str) -> str:
    """Short hash of a unit's sources under csrc/ (kernels, helpers, launch logic): names the
    exact device code and launch configuration.  The public header holds declarations only
    and is left out, so documenting a new entry point does not change the hash."""
    h = hashlib.sha256()
    for path in dependency_files(unit):
        if not path.startswith(CSRC):
            continue
        with open(path, "rb") as f:
            h.update(os.path.basename(path).encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def _object(unit: str) -> str:
    return os.path.join(OBJDIR, unit.replace(".cu", ".o"))


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(unit: str, verbose: bool) -> str:
    obj = _object(unit)
    tmp = obj + ".tmp%d" % os.getpid()
    cmd = [NVCC] + CFLAGS + (["-Xptxas", "-v"] if verbose else []) + [
        "-c", os.path.join(CSRC, unit), "-o", tmp]
    subprocess.check_call(cmd)
    os.replace(tmp, obj)
    return obj


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    return not any(_stale(LIB, dependency_files(u)) for u in UNITS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(OBJDIR, exist_ok=True)
    todo = [u for u in UNITS if force or _stale(_object(u), dependency_files(u))]
    with concurrent.futures.ThreadPoolExecutor(max_workers=max(1, len(todo))) as pool:
        for f in [pool.submit(_compile, u, verbose) for u in todo]:
            f.result()
    tmp = LIB + ".tmp%d" % os.getpid()
    subprocess.check_call([NVCC] + ARCH + ["-shared", "-o", tmp] + [_object(u) for u in UNITS])
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
