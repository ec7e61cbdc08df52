"""Build step for libdf11.so: the sm_100a decode kernels, their C ABI, and the
host and device format builders, compiled in-tree with nvcc (no GPU needed to build).

    python -m huffman_decode_df11_b200._build [--force]
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libdf11.so")
SOURCES = [os.path.join(CSRC, "df11_decode.cu"), os.path.join(CSRC, "df11_gpu_build.cu"),
           os.path.join(CSRC, "df11_build.cpp")]
HEADERS = [os.path.join(INCLUDE, "df11.h"), os.path.join(CSRC, "df11_codebook.h"),
           os.path.join(CSRC, "df11_device_check.h")]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in SOURCES + HEADERS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC,-O3,-pthread", "-I", INCLUDE,
           "--expt-relaxed-constexpr", *SOURCES, "-o", tmp, "-lpthread"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
