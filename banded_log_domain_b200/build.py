"""Builds libsinkhorn_attn.so in-tree with nvcc for sm_100a.

    python -m banded_log_domain_b200.build [--force]
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libsinkhorn_attn.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-I", os.path.join(ROOT, "include"),
]


def sources():
    return [os.path.join(CSRC, "sinkhorn_attn.cu")]


def deps():
    return (glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
            glob.glob(os.path.join(ROOT, "include", "*.h")))


DEBUG_LIB = os.path.join(PKG, "libsinkhorn_attn_debug.so")


def stale_lib(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in deps())


def build(force: bool = False, verbose: bool = False) -> str:
    """Builds the library and its bounds-checked debug twin (-DSA_DEBUG)."""
    for lib, extra in ((LIB, []), (DEBUG_LIB, ["-DSA_DEBUG"])):
        if force or stale_lib(lib):
            tmp = lib + f".tmp{os.getpid()}"
            cmd = [NVCC, *FLAGS, *extra, "-o", tmp, *sources()]
            if verbose:
                print(" ".join(cmd), flush=True)
            subprocess.check_call(cmd)
            os.replace(tmp, lib)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(LIB)
