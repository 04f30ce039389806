"""Seeded synthetic inputs for the W4A16 linear layer.

This package draws inputs only (FP32 weights, BF16 activations with salient
channels); it holds none of the quantisation or matmul arithmetic.  It is the
one module shared by the CUDA library's tests/benchmark and by the FP64 oracle.

Generator: counter-based SplitMix64 (Steele, Lea & Flood, OOPSLA 2014) feeding
Box-Muller (Box & Muller, 1958), defined once in ``synth_core.h`` and compiled
for the host (``synth.c``) and the device (``synth_dev.cu``) so both produce
identical bits for any element index.

Recipe (values are the workloads' stated distributions):
  * W[n, k] = fp32(sigma * normal(key(seed, tag_w), n*K + k)), sigma = 0.02
  * salient channels: round(1% of K) distinct input channels chosen by a
    partial Fisher-Yates shuffle keyed by (seed, TAG_OUTLIERS), the same for
    every row of X
  * X[m, k] = bf16_rne(normal(key(seed, TAG_X), m*K + k) * (20 if k salient else 1))
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
HOST_LIB = os.path.join(_HERE, "libsynth.so")
DEV_LIB = os.path.join(_HERE, "libsynth_dev.so")

TAG_W = 1
TAG_X = 2
TAG_OUTLIERS = 3
TAG_W_STACK = 16  # + matrix index inside a layer of the 80-layer stack

SIGMA_W = 0.02
OUTLIER_FRACTION = 0.01
OUTLIER_MULT = 20.0

_host = None
_dev = None


def build_host(force: bool = False) -> str:
    src = [os.path.join(_HERE, "synth.c")]
    if force or not os.path.exists(HOST_LIB) or os.path.getmtime(HOST_LIB) < max(
        os.path.getmtime(p) for p in src + [os.path.join(_HERE, "synth_core.h")]
    ):
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
             "-o", HOST_LIB] + src + ["-lm"]
        )
    return HOST_LIB


def build_device(force: bool = False) -> str:
    src = os.path.join(_HERE, "synth_dev.cu")
    if force or not os.path.exists(DEV_LIB) or os.path.getmtime(DEV_LIB) < max(
        os.path.getmtime(src), os.path.getmtime(os.path.join(_HERE, "synth_core.h"))
    ):
        subprocess.check_call(
            ["nvcc", "-O3", "-std=c++17", "-fmad=false", "-gencode", "arch=compute_100a,code=sm_100a",
             "-Xcompiler", "-fPIC", "-shared", "-o", DEV_LIB, src]
        )
    return DEV_LIB


def _lib():
    global _host
    if _host is None:
        build_host()
        lib = ctypes.CDLL(HOST_LIB)
        u64, i64, dbl = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double
        vp = ctypes.c_void_p
        lib.synth_key.argtypes = [u64, u64]
        lib.synth_key.restype = u64
        lib.synth_draw.argtypes = [u64, u64]
        lib.synth_draw.restype = u64
        lib.synth_ln.argtypes = [dbl]
        lib.synth_ln.restype = dbl
        lib.synth_cos2pi.argtypes = [dbl]
        lib.synth_cos2pi.restype = dbl
        lib.synth_normal.argtypes = [u64, u64]
        lib.synth_normal.restype = dbl
        lib.synth_fill_normal_f32.argtypes = [u64, u64, u64, i64, dbl, vp]
        lib.synth_fill_normal_f32.restype = None
        lib.synth_fill_normal_rows_f32.argtypes = [u64, u64, i64, vp, i64, dbl, vp]
        lib.synth_fill_normal_rows_f32.restype = None
        lib.synth_bf16_bits.argtypes = [dbl]
        lib.synth_bf16_bits.restype = ctypes.c_uint16
        lib.synth_outlier_channels.argtypes = [u64, u64, i64, i64, vp, vp]
        lib.synth_outlier_channels.restype = None
        lib.synth_fill_activations_bf16.argtypes = [u64, u64, i64, i64, vp, i64, dbl, vp, vp]
        lib.synth_fill_activations_bf16.restype = None
        lib.synth_threads.argtypes = []
        lib.synth_threads.restype = ctypes.c_int
        _host = lib
    return _host


def _dev_lib():
    global _dev
    if _dev is None:
        build_device()
        lib = ctypes.CDLL(DEV_LIB)
        lib.synth_dev_fill_normal_f32.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64,
                                                  ctypes.c_int64, ctypes.c_double, ctypes.c_void_p,
                                                  ctypes.c_void_p]
        lib.synth_dev_fill_normal_f32.restype = ctypes.c_int
        _dev = lib
    return _dev


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def n_outliers(K: int) -> int:
    """round(1% of K), halves up (41, 51, 82, 256, 287 for the workloads' K)."""
    return (K + 50) // 100


def key(seed: int, tag: int) -> int:
    return int(_lib().synth_key(seed, tag))


def normal(seed: int, tag: int, i: int) -> float:
    return float(_lib().synth_normal(key(seed, tag), i))


def ln(u: float) -> float:
    return float(_lib().synth_ln(u))


def cos2pi(u: float) -> float:
    return float(_lib().synth_cos2pi(u))


def bf16_bits(x: float) -> int:
    return int(_lib().synth_bf16_bits(float(x)))


def weights_f32(seed: int, tag: int, N: int, K: int, sigma: float = SIGMA_W) -> np.ndarray:
    out = np.empty((N, K), dtype=np.float32)
    _lib().synth_fill_normal_f32(seed, tag, 0, N * K, sigma, _ptr(out))
    return out


def weight_rows_f32(seed: int, tag: int, K: int, rows, sigma: float = SIGMA_W) -> np.ndarray:
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.empty((rows.size, K), dtype=np.float32)
    _lib().synth_fill_normal_rows_f32(seed, tag, K, _ptr(rows), rows.size, sigma, _ptr(out))
    return out


def outlier_channels(seed: int, K: int, n_out: int | None = None) -> np.ndarray:
    n_out = n_outliers(K) if n_out is None else n_out
    ch = np.empty(n_out, dtype=np.int64)
    perm = np.empty(K, dtype=np.int64)
    _lib().synth_outlier_channels(seed, TAG_OUTLIERS, K, n_out, _ptr(ch), _ptr(perm))
    return ch


def activations_bf16(seed: int, M: int, K: int, n_out: int | None = None,
                     mult: float = OUTLIER_MULT) -> np.ndarray:
    """X as BF16 bit patterns (uint16), shape [M, K]."""
    ch = outlier_channels(seed, K, n_out)
    X = np.empty((M, K), dtype=np.uint16)
    flags = np.empty(K, dtype=np.uint8)
    _lib().synth_fill_activations_bf16(seed, TAG_X, M, K, _ptr(ch), ch.size, mult, _ptr(X), _ptr(flags))
    return X


def fill_weights_device(seed: int, tag: int, out_ptr: int, count: int, offset: int = 0,
                        sigma: float = SIGMA_W, stream: int = 0) -> None:
    """Fill ``count`` FP32 values at device address ``out_ptr`` (same bits as weights_f32)."""
    rc = _dev_lib().synth_dev_fill_normal_f32(seed, tag, offset, count, sigma, out_ptr, stream)
    if rc != 0:
        raise RuntimeError(f"synth device fill failed (code {rc})")


def host_threads() -> int:
    return int(_lib().synth_threads())
