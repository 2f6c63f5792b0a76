"""Builds libqlora.so in-tree with nvcc for sm_100a (B200).

Run as ``python bit_nf4_quantized_encode_b200/build.py`` (a script, so that a
stale library is never loaded while rebuilding it) or call ``build()``.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libqlora.so")
SOURCES = ["api.cu", "codec.cu", "gemm.cu", "gemv.cu", "lora.cu", "noalloc.cu", "selftest.cu", "nf4_tables.cpp"]
HEADERS = ["codec.h", "gemm.h", "gemv.h", "internal.h", "lora.h", "nf4_device.cuh", "nf4_tables.h", "sm100_ptx.cuh"]


def _newest_input() -> float:
    paths = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "qlora.h")]
    return max(os.path.getmtime(p) for p in paths)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= _newest_input():
        return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-shared", "-Xcompiler", "-fPIC,-fvisibility=hidden", "-I", INCLUDE,
           "-diag-suppress", "177"]
    cmd += [os.path.join(CSRC, f) for f in SOURCES]
    cmd += ["-o", tmp]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
