"""Builds libfnl.so (the C-ABI CUDA library) in-tree for sm_100a.

    python -m transformer_layer_residual_b200.build [--verbose] [--force] [--debug]

The library is one translation unit (csrc/fnl.cu) compiled by nvcc with the
CUDA runtime linked statically, so the .so depends only on the driver.
--debug builds libfnl_debug.so instead: the same code with FNL_DEBUG_CHECKS,
which checks every output store against its buffer (an out-of-range store is
skipped and reported through fnl_check as device status 8). The binding loads
it when FNL_LIBRARY=debug is set.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libfnl.so")
LIB_DEBUG = os.path.join(PKG, "libfnl_debug.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2",
    "--expt-relaxed-constexpr",
    "-shared",
]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list:
    return [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC))]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    deps = sources() + [os.path.join(INCLUDE, "fnl.h"), os.path.abspath(__file__)]
    return all(os.path.getmtime(d) <= t for d in deps)


def build(verbose: bool = False, force: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and up_to_date(lib):
        return lib
    cmd = [nvcc()] + NVCC_FLAGS + (["-DFNL_DEBUG_CHECKS"] if debug else []) + \
        ["-I", INCLUDE, "-I", CSRC, "-o", lib + ".tmp", os.path.join(CSRC, "fnl.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose:
        sys.stdout.write(res.stdout + res.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force="--force" in sys.argv, debug="--debug" in sys.argv))
