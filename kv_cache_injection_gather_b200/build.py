"""Builds libinjectstore.so in-tree for sm_100a (nvcc, no JIT cache).

    python -m kv_cache_injection_gather_b200.build [--force] [--verbose]
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libinjectstore.so")
SOURCES = [os.path.join(CSRC, "inject_store.cu")]
DEPS = SOURCES + [os.path.join(CSRC, "inject_kernels.cuh"),
                  os.path.join(ROOT, "include", "inject_store.h")]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_command(out: str, verbose: bool = False) -> list[str]:
    cmd = ["nvcc", "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC,-O2", "-lineinfo",
           *ARCH, "-I", os.path.join(ROOT, "include"), "-I", CSRC, "-o", out, *SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def build(force: bool = False, verbose: bool = False) -> str:
    stale = not os.path.exists(LIB) or any(os.path.getmtime(LIB) < os.path.getmtime(d) for d in DEPS)
    if force or stale or verbose:
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.run(nvcc_command(tmp, verbose), check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    print(LIB)
