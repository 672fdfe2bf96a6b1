"""Build libsq.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc.

    python -m w8a8_post_quantization_calibrate_b200.build [--force] [--verbose] [--debug]

The library is one translation unit (csrc/sq_lib.cu includes the others) built
with -gencode arch=compute_100a,code=sm_100a and -lineinfo. No GPU is needed to
build: nvcc cross-compiles.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libsq.so")
# the same sources with -DSQ_DEBUG: index checks before the kernels' unguarded
# stores, reported through the status word (never a trap)
LIB_DEBUG = os.path.join(PKG, "libsq_debug.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(CSRC, "*.h")) + [os.path.join(INCLUDE, "sq.h")])


def up_to_date(lib: str) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and up_to_date(lib):
        return lib
    cmd = [nvcc(), "-std=c++17", "-O3", "-lineinfo", *ARCH_FLAGS,
           "-Xcompiler", "-fPIC", "-shared", "-I", INCLUDE, "-I", CSRC, *(["-DSQ_DEBUG"] if debug else []),
           "-o", lib + ".tmp", os.path.join(CSRC, "sq_lib.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError(f"nvcc failed building {os.path.basename(lib)}")
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, debug="--debug" in sys.argv))
