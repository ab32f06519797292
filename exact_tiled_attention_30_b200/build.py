"""Builds the sm_100a shared library ``libfa2_b200.so`` in place with nvcc.

The library exposes only the C ABI of ``include/fa2.h``; the CUDA runtime is
linked statically and the driver's tensor-map encoder is resolved at run time,
so the library loads (and its argument checks run) on machines without a GPU.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libfa2_b200.so")
#: test-only build of the same sources: 20 ms wait limit and the planted-stall
#: hook (fa2_debug_set_stall) that the timeout test uses; never loaded by the
#: package itself
TEST_HOOKS_LIB = os.path.join(PKG, "libfa2_b200_testhooks.so")
TEST_HOOKS_FLAGS = ["-DFA2_TEST_HOOKS", "-DFA2_WAIT_LIMIT_NS=20000000ull"]
SOURCES = [os.path.join(CSRC, "fa2_api.cu")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "--expt-relaxed-constexpr",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "-shared", "--cudart", "static",
]


def _deps():
    files = list(SOURCES)
    for name in os.listdir(CSRC):
        if name.endswith((".cuh", ".h")):
            files.append(os.path.join(CSRC, name))
    files.append(os.path.join(INCLUDE, "fa2.h"))
    return files


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in _deps())


def build(force: bool = False, verbose: bool = False, extra_flags=(), lib: str = LIB) -> str:
    """Compile the library if any source is newer than it; returns its path."""
    if not force and not needs_build(lib):
        return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, *extra_flags, f"-I{INCLUDE}", f"-I{CSRC}", *SOURCES, "-o", tmp]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def build_test_hooks(force: bool = False, verbose: bool = False) -> str:
    """Compile the test-hooks library (TEST_HOOKS_LIB); returns its path."""
    return build(force=force, verbose=verbose, extra_flags=TEST_HOOKS_FLAGS, lib=TEST_HOOKS_LIB)


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra_flags=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
    build_test_hooks(force="--force" in sys.argv, verbose=True)
