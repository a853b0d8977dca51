"""Build libflint.so in-tree: nvcc for sm_100a, no JIT, no torch dependency.

    python -m long_context_decode_flash_b200.build [--force] [--ptxas-info]
        [--debug-checks] [--trace] [--nvtx] [--out PATH]
    python -m long_context_decode_flash_b200.build --hooks   # libflint_hooks.so

--debug-checks: the kernels' bounds and alignment self-checks; --trace: the
decode kernel's per-CTA timeline stamps; --nvtx: NVTX ranges around every
entry point.  Variants are meant for --out paths next to the release build.
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
# The build the time-out tests load: self-checks, the stall hooks and a 5 ms
# wait limit, so that a wait on a stage nobody arms runs out quickly.
HOOKS_LIB = os.path.join(HERE, "libflint_hooks.so")
HOOKS_WAIT_LIMIT_NS = 5_000_000
SOURCES = ["flint_abi.cu", "flint_decode.cu", "flint_prep.cu", "flint_prefill.cu", "flint_prefill_prep.cu", "flint_cp.cu", "flint_plan.cpp", "flint_noalloc.cu"]
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


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build_hooks(force: bool = False, verbose: bool = False) -> str:
    """libflint_hooks.so: the library with FLINT_DEBUG_CHECKS, FLINT_TEST_HOOKS
    (flint_test_stall_decode / flint_test_stall_prefill) and a short wait
    limit, for the tests of the kernels' time-out path."""
    if not force and up_to_date(HOOKS_LIB):
        return HOOKS_LIB
    return build(force=True, verbose=verbose, debug_checks=True, out=HOOKS_LIB,
                 defines=["FLINT_TEST_HOOKS", f"FLINT_WAIT_LIMIT_NS={HOOKS_WAIT_LIMIT_NS}ull"])


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False,
          debug_checks: bool = False, trace: bool = False, out: str | None = None,
          defines=()) -> str:
    """debug_checks compiles the kernels' self-checks in (bounds and alignment
    checks that record the first failure in dev_err[2..7] and skip the access).
    trace compiles the decode kernel's timeline stamps in (FLINT_TRACE) and
    exports flint_trace_read / flint_trace_clear.  out: write the library
    there instead of the package's libflint.so (the variants above are meant
    for a separate path)."""
    lib = out or LIB
    if not force and not debug_checks and not trace and out is None and not defines and up_to_date():
        return LIB
    tmp = lib + f".{os.getpid()}.tmp"
    cmd = [nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
           "-I", os.path.join(ROOT, "include"), "-o", tmp]
    if ptxas_info:
        cmd += ["-Xptxas", "-v"]
    if debug_checks:
        cmd += ["-DFLINT_DEBUG_CHECKS"]
    if trace:
        cmd += ["-DFLINT_TRACE"]
    cmd += [f"-D{d}" for d in defines]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    out = sys.argv[sys.argv.index("--out") + 1] if "--out" in sys.argv else None
    if "--hooks" in sys.argv:
        build_hooks(force="--force" in sys.argv, verbose=True)
    else:
        build(force="--force" in sys.argv, verbose=True, ptxas_info="--ptxas-info" in sys.argv,
              debug_checks="--debug-checks" in sys.argv, trace="--trace" in sys.argv, out=out,
              defines=["FLINT_NVTX"] if "--nvtx" in sys.argv else ())
