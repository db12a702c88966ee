"""Builds the CUDA library libllama_attn.so in-tree for sm_100a (nvcc)."""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "llama_attn.cu")
LIB = os.path.join(PKG, "libllama_attn.so")
INCLUDE = os.path.join(ROOT, "include")


def sources():
    csrc = os.path.join(PKG, "csrc")
    files = [os.path.join(csrc, f) for f in os.listdir(csrc) if f.endswith((".cu", ".cuh"))]
    return files + [os.path.join(INCLUDE, "llama_attn.h")]


def nvcc_command(out: str = LIB, extra=()):
    return ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
            "-shared", "-Xcompiler", "-fPIC", "-I" + INCLUDE, *extra, "-o", out, SRC]


def build(force: bool = False, verbose: bool = False) -> str:
    stale = force or not os.path.exists(LIB) or any(
        os.path.getmtime(f) > os.path.getmtime(LIB) for f in sources())
    if stale:
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = nvcc_command(tmp, ["-Xptxas", "-v"] if verbose else [])
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
