"""Build libulysses.so (the C-ABI library) in-tree with nvcc for sm_100a.

Usage: python -m ulysses_sequence_attention_repack_b200.build [--debug]

--debug builds libulysses_debug.so instead: the same library compiled with
-DULYSSES_DEBUG, whose repack, prologue, push and attention-epilogue kernels
range-check every computed global offset (an access outside its buffer is
skipped and reported through the device error word).  Select it at run time
with ULYSSES_LIBRARY=<path> (see _lib.load).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libulysses.so")
# test hooks (device helpers run on their own) live in a library of their own,
# so the product library exports only what include/ulysses.h declares
SELFTEST_LIB = os.path.join(PKG, "libulysses_selftest.so")
DEBUG_LIB = os.path.join(PKG, "libulysses_debug.so")
SOURCES = ["api.cpp", "repack.cu", "prologue.cu", "attn_fwd.cu", "attn_bwd.cu", "noalloc.cu", "transport.cu"]
SELFTEST_SOURCES = ["selftest.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps():
    return [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [
        os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))]


def sources_newer_than_lib(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(d) > t for d in _deps() if os.path.exists(d))


def _compile(out: str, sources, debug: bool, verbose: bool) -> None:
    cmd = [nvcc_path(), "-shared", "-Xcompiler", "-fPIC", "-std=c++17", "-O3", "-lineinfo", *ARCH,
           "-I", os.path.join(ROOT, "include"), "-o", out + ".tmp"]
    if debug:
        cmd += ["-DULYSSES_DEBUG"]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in sources]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)


def build(debug: bool = False, verbose: bool = False) -> str:
    """Compile the product library and the test-hook library (or, with
    debug, the bounds-checked library); returns the library's path."""
    if debug:
        _compile(DEBUG_LIB, SOURCES, True, verbose)
        return DEBUG_LIB
    _compile(LIB, SOURCES, False, verbose)
    _compile(SELFTEST_LIB, SELFTEST_SOURCES, False, verbose)
    return LIB


def ensure_debug_built() -> str:
    if sources_newer_than_lib(DEBUG_LIB):
        build(debug=True)
    return DEBUG_LIB


def ensure_built() -> str:
    if sources_newer_than_lib(LIB) or sources_newer_than_lib(SELFTEST_LIB):
        build()
    return LIB


if __name__ == "__main__":
    print(build(debug="--debug" in sys.argv, verbose="-v" in sys.argv))
