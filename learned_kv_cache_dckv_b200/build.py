"""Build the in-tree CUDA library libdckv_b200.so for sm_100a with nvcc.

Usage: python -m learned_kv_cache_dckv_b200.build [--force] [--verbose-ptxas]
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libdckv_b200.so")
SOURCES = [os.path.join(HERE, "csrc", "dckv.cu")]
DEPS = SOURCES + [os.path.join(HERE, "csrc", f) for f in os.listdir(os.path.join(HERE, "csrc"))] + [
    os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def command(out: str = LIB, ptxas_verbose: bool = False) -> list[str]:
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
           "-I", os.path.join(ROOT, "include"), "-o", out] + SOURCES
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    if not force and os.path.exists(LIB):
        t = os.path.getmtime(LIB)
        if all(os.path.getmtime(d) <= t for d in DEPS if os.path.exists(d)):
            return LIB
    tmp = LIB + f".{os.getpid()}.tmp"
    subprocess.check_call(command(tmp, ptxas_verbose))
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, ptxas_verbose="--verbose-ptxas" in sys.argv)
    print(LIB)
