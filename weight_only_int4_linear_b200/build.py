"""Build the in-tree CUDA library libw4a16.so for sm_100a (nvcc, no JIT cache).

Usage: python -m weight_only_int4_linear_b200.build [--force]
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libw4a16.so")
OBJ_DIR = os.path.join(PKG, "_build")
SOURCES = ["api.cu", "runtime.cu", "pack.cu", "gemv.cu", "gemv_mt.cu", "gemv_bf.cu", "gemv_sub.cu", "gemm.cu",
           "noalloc.cu", "w8.cu"]
HEADERS = ["common.cuh", "sm100.cuh", "decode_units.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-I", os.path.join(ROOT, "include"),
]


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(OBJ_DIR, exist_ok=True)
    headers = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", h) for h in ("w4a16.h", "w8a16.h")]
    objs = []
    for src in SOURCES:
        path = os.path.join(CSRC, src)
        obj = os.path.join(OBJ_DIR, src.replace(".cu", ".o"))
        objs.append(obj)
        if force or _stale(obj, [path] + headers):
            cmd = ["nvcc"] + NVCC_FLAGS + ["-c", path, "-o", obj]
            if verbose:
                cmd += ["-Xptxas", "-v"]
            subprocess.check_call(cmd)
    if force or _stale(LIB, objs):
        subprocess.check_call(["nvcc", "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", LIB] + objs +
                              ["-lcudart"])
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
