"""Build libfa.so (the C-ABI attention library) in-tree with nvcc for sm_100a.

Usage: ``python -m io_aware_exact_23_b200.build [--force] [-v]``.
The library is written next to this file so that it travels with the source
tree; nothing is installed into site-packages.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libfa.so")
# Standard-attention baseline (cuBLAS GEMMs + its own row kernels), kept out of libfa.so.
VANILLA_LIB = os.path.join(PKG, "libfa_vanilla.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libfa.so")
    return cand


def sources():
    return [os.path.join(CSRC, "fa_api.cu")]


def deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + [os.path.join(INCLUDE, "fa.h")]


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in deps())


def vanilla_deps():
    return [os.path.join(CSRC, "vanilla.cu"), os.path.join(INCLUDE, "fa.h"), os.path.join(INCLUDE, "fa_vanilla.h")]


def build_vanilla(force: bool = False, verbose: bool = False) -> str:
    """Compile libfa_vanilla.so (links cuBLAS)."""
    if not force and os.path.exists(VANILLA_LIB) and all(
            os.path.getmtime(p) <= os.path.getmtime(VANILLA_LIB) for p in vanilla_deps()):
        return VANILLA_LIB
    tmp = VANILLA_LIB + f".tmp{os.getpid()}"
    cmd = [nvcc_path(), *ARCH, "-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
           "-I", INCLUDE, os.path.join(CSRC, "vanilla.cu"), "-lcublas", "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, VANILLA_LIB)
    return VANILLA_LIB


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    if not force and not needs_build():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc_path(), *ARCH, "-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
           "-I", INCLUDE, "-I", CSRC, *extra, *sources(), "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true", help="print the command and ptxas resource usage")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
    print(build_vanilla(force=a.force, verbose=a.verbose))
    sys.exit(0)
