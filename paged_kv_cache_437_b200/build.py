"""Build libpkv.so in-tree with nvcc for sm_100a (B200).

    python paged_kv_cache_437_b200/build.py [--verbose]

The shared library lands next to this file; the Python binding loads it from
there and nowhere else.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libpkv.so")
SOURCES = [os.path.join(CSRC, "pkv_cuda.cu"), os.path.join(CSRC, "allocator.cpp"),
           os.path.join(CSRC, "scheduler.cpp")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("decode.cuh", "mq_attention.cuh", "ptx.cuh")] + [os.path.join(INCLUDE, "pkv.h")]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "--use_fast_math",
    "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
]


def build(force: bool = False, verbose: bool = False, out: str = LIB, extra=None) -> str:
    if not force and os.path.exists(out):
        newest = max(os.path.getmtime(p) for p in DEPS)
        if os.path.getmtime(out) >= newest and not extra:
            return out
    cmd = [NVCC, *FLAGS, "-I", INCLUDE, "-I", CSRC, *(extra or []), *SOURCES, "-o", out]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
