"""Build libflint.so in-tree: nvcc for sm_100a, no JIT, no torch dependency.

    python -m long_context_decode_flash_b200.build
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libflint.so")
SOURCES = ["flint_abi.cu", "flint_decode.cu", "flint_prep.cu", "flint_prefill.cu", "flint_cp.cu", "flint_plan.cpp", "flint_noalloc.cu"]
HEADERS = ["flint_internal.h", "flint_device.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _inputs():
    return ([os.path.join(CSRC, s) for s in SOURCES + HEADERS] +
            [os.path.join(ROOT, "include", "flint.h")])


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False,
          debug_checks: bool = False) -> str:
    """debug_checks compiles the kernels' self-checks in (bounds and alignment
    checks that record the first failure in dev_err[2..7] and skip the access)."""
    if not force and not debug_checks and up_to_date():
        return LIB
    tmp = LIB + f".{os.getpid()}.tmp"
    cmd = [nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
           "-I", os.path.join(ROOT, "include"), "-o", tmp]
    if ptxas_info:
        cmd += ["-Xptxas", "-v"]
    if debug_checks:
        cmd += ["-DFLINT_DEBUG_CHECKS"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, ptxas_info="--ptxas-info" in sys.argv,
          debug_checks="--debug-checks" in sys.argv)
