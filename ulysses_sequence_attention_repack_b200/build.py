"""Build libulysses.so (the C-ABI library) in-tree with nvcc for sm_100a.

Usage: python -m ulysses_sequence_attention_repack_b200.build [--debug]
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
SOURCES = ["api.cpp", "repack.cu", "prologue.cu", "attn_fwd.cu", "attn_bwd.cu", "selftest.cu", "noalloc.cu",
           "transport.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources_newer_than_lib() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(ROOT, "include", "ulysses.h")]
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def build(debug: bool = False, verbose: bool = False) -> str:
    """Compile every source into one shared library; returns its path."""
    cmd = [nvcc_path(), "-shared", "-Xcompiler", "-fPIC", "-std=c++17", "-O3", "-lineinfo", *ARCH,
           "-I", os.path.join(ROOT, "include"), "-o", LIB + ".tmp"]
    if debug:
        cmd += ["-DULYSSES_DEBUG"]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


def ensure_built() -> str:
    if sources_newer_than_lib():
        build()
    return LIB


if __name__ == "__main__":
    build(debug="--debug" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
