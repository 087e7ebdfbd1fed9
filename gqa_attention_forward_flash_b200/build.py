"""Builds libgqa_attn.so (the CUDA kernels + C ABI) in-tree for sm_100a.

    python -m gqa_attention_forward_flash_b200.build [--verbose]

nvcc cross-compiles without a GPU.  ``--verbose`` adds ``-Xptxas -v`` (registers,
spills and shared memory per kernel).
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libgqa_attn.so")
SOURCES = [os.path.join(CSRC, "gqa_attn.cu")]
HEADERS = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))] + \
    [os.path.join(ROOT, "include", "gqa_attn.h")]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.sep not in c or os.path.exists(c)):
            return c
    return "nvcc"


def command(out: str = LIB, verbose: bool = False) -> list:
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
           "-o", out] + SOURCES
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    return cmd


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in SOURCES + HEADERS)


def build(force: bool = False, verbose: bool = False) -> str:
    if force or verbose or stale():
        tmp = LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(command(tmp, verbose))
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
