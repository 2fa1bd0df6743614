"""Build the CUDA library (libmoe.so) in-tree for sm_100a.

    python mixture_experts_ffn_11_b200/build.py [--force] [--verbose]

Run it by path (or load it with load_build_module below): importing the package itself loads libmoe.so,
which is what this script produces.

The library is one translation unit (csrc/moe.cu plus the kernel headers it includes) compiled by nvcc
into a shared object next to this file, so it travels with the source tree.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmoe.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    files = [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith((".cu", ".cuh"))]
    return files + [os.path.join(INCLUDE, "moe.h")]


def nvcc_command(out: str = LIB, verbose: bool = False, extra=()):
    cmd = ["nvcc", "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-lineinfo", *ARCH,
           "-I", INCLUDE, "-I", CSRC, os.path.join(CSRC, "moe.cu"), "-o", out, *extra]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def load_build_module():
    """This module, loaded by file path without importing the package (usable before libmoe.so exists)."""
    import importlib.util

    spec = importlib.util.spec_from_file_location("_moe_build", os.path.abspath(__file__))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def build(force: bool = False, verbose: bool = False) -> str:
    stale = force or not os.path.exists(LIB) or any(os.path.getmtime(s) > os.path.getmtime(LIB) for s in sources())
    if stale:
        subprocess.check_call(nvcc_command(verbose=verbose))
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    print(LIB)
