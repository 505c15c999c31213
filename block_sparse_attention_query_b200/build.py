"""Build libbsa.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc.

    python -m block_sparse_attention_query_b200.build [--force]

nvcc cross-compiles without a GPU. The library links the CUDA runtime statically, so it
loads next to any PyTorch build.
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
LIB = os.path.join(PKG, "libbsa.so")
# Test-only variant: bounded waits of about 10 ms instead of 2 s, and a hook that makes the
# attention kernel take its timeout path (tests/test_wait_timeout.py). Never loaded by the
# package itself.
WAITTEST_LIB = os.path.join(PKG, "libbsa_waittest.so")
WAITTEST_FLAGS = ["-DBSA_TEST_HOOKS", "-DBSA_WAIT_LIMIT_CYCLES=20000000LL"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: set NVCC or put the CUDA toolkit on PATH")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(ROOT, "include", "bsa.h")])


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in _sources())


def _compile(lib: str, extra, verbose: bool) -> str:
    units = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    tmp = lib + ".tmp"
    cmd = [_nvcc(), *NVCC_FLAGS, *extra, "-I", os.path.join(ROOT, "include"), "-o", tmp, *units]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not needs_build(LIB):
        return LIB
    return _compile(LIB, [], verbose)


def build_wait_test(force: bool = False, verbose: bool = False) -> str:
    """The test-only variant with short waits and the timeout hook."""
    if not force and not needs_build(WAITTEST_LIB):
        return WAITTEST_LIB
    return _compile(WAITTEST_LIB, WAITTEST_FLAGS, verbose)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
    print(build_wait_test(force="--force" in sys.argv, verbose=True))
