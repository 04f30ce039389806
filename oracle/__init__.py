"""FP64 CPU oracle for the W4A16 weight-only linear layer (ctypes loader).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The product path never
imports this package, and this package never imports the product package.

The arithmetic lives in ``oracle.c`` (plain C, binary64, OpenMP over rows);
this file only compiles it with gcc and marshals numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(_HERE, "liboracle.so")
SRC = os.path.join(_HERE, "oracle.c")
G = 128

OK = 0
ERR_ARG = 1
ERR_SHAPE = 3
ERR_NONFINITE = 7
ERR_ZERO_RANGE = 8

_lib = None


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                               "-shared", "-fPIC", "-o", LIB, SRC, "-lm"])
    return LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB)
        i64, vp = ctypes.c_int64, ctypes.c_void_p
        L.orc_threads.argtypes = []
        L.orc_threads.restype = ctypes.c_int
        L.orc_bf16_value.argtypes = [ctypes.c_uint16]
        L.orc_bf16_value.restype = ctypes.c_double
        L.orc_bf16_round.argtypes = [ctypes.c_double]
        L.orc_bf16_round.restype = ctypes.c_uint16
        L.orc_pack_codes.argtypes = [vp, i64, i64, vp]
        L.orc_pack_codes.restype = None
        L.orc_quantize_pack.argtypes = [vp, i64, i64, vp, vp, vp, vp]
        L.orc_quantize_pack.restype = ctypes.c_int
        L.orc_quantize_pack_sym.argtypes = [vp, i64, i64, vp, vp, vp, vp]
        L.orc_quantize_pack_sym.restype = ctypes.c_int
        L.orc_quantize_pack_g.argtypes = [vp, i64, i64, i64, ctypes.c_int, vp, vp, vp, vp]
        L.orc_quantize_pack_g.restype = ctypes.c_int
        L.orc_dequant_g.argtypes = [vp, vp, vp, i64, i64, i64, vp]
        L.orc_dequant_g.restype = None
        L.orc_linear_g.argtypes = [vp, i64, i64, vp, vp, vp, i64, i64, vp]
        L.orc_linear_g.restype = None
        L.orc_unpack.argtypes = [vp, i64, i64, vp]
        L.orc_unpack.restype = None
        L.orc_dequant.argtypes = [vp, vp, vp, i64, i64, vp]
        L.orc_dequant.restype = None
        L.orc_dequant_bf16.argtypes = [vp, vp, vp, i64, i64, vp]
        L.orc_dequant_bf16.restype = None
        L.orc_linear.argtypes = [vp, i64, i64, vp, vp, vp, i64, vp]
        L.orc_linear.restype = None
        L.orc_linear_sampled.argtypes = [vp, i64, i64, vp, vp, vp, i64, vp, i64, vp, i64, vp]
        L.orc_linear_sampled.restype = None
        L.orc_awq_scale_weights.argtypes = [vp, vp, i64, i64, vp]
        L.orc_awq_scale_weights.restype = None
        L.orc_awq_scale_activations.argtypes = [vp, vp, i64, i64, vp]
        L.orc_awq_scale_activations.restype = None
        L.orc_w8_quantize.argtypes = [vp, i64, i64, vp, vp, vp]
        L.orc_w8_quantize.restype = ctypes.c_int
        L.orc_w8_linear.argtypes = [vp, i64, i64, vp, vp, i64, vp]
        L.orc_w8_linear.restype = None
        L.orc_renorm.argtypes = [vp, i64, i64, vp, vp]
        L.orc_renorm.restype = None
        _lib = L
    return _lib


def _p(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def threads() -> int:
    return int(lib().orc_threads())


def bf16_value(bits: int) -> float:
    return float(lib().orc_bf16_value(bits))


def bf16_round(x: float) -> int:
    return int(lib().orc_bf16_round(float(x)))


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """BF16 bit patterns -> float64 values (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def quantize_pack(W: np.ndarray, with_clipped: bool = False, symmetric: bool = False):
    """W float32 [N, K] -> (status, qweight u32 [N, K/8], scales bf16-bits u16 [N, K/128],
    zeros i32 [N, K/128][, clipped u8 [N, K]]).  symmetric=True: signed codes
    q = clamp(rint(w/s), -8, 7) with s = bf16(max|w|/7), stored as q + 8 with zero point 8."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    qw = np.zeros((N, K // 8), dtype=np.uint32)
    sc = np.zeros((N, max(K // G, 1)), dtype=np.uint16)
    z = np.zeros((N, max(K // G, 1)), dtype=np.int32)
    cl = np.zeros((N, K), dtype=np.uint8) if with_clipped else None
    fn = lib().orc_quantize_pack_sym if symmetric else lib().orc_quantize_pack
    st = fn(_p(W), N, K, _p(qw), _p(sc), _p(z), _p(cl) if cl is not None else None)
    if with_clipped:
        return st, qw, sc, z, cl
    return st, qw, sc, z


def pack_codes(codes: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    N, K = codes.shape
    qw = np.zeros((N, K // 8), dtype=np.uint32)
    lib().orc_pack_codes(_p(codes), N, K, _p(qw))
    return qw


def unpack(qweight: np.ndarray, K: int) -> np.ndarray:
    qweight = np.ascontiguousarray(qweight, dtype=np.uint32)
    N = qweight.shape[0]
    codes = np.zeros((N, K), dtype=np.uint8)
    lib().orc_unpack(_p(qweight), N, K, _p(codes))
    return codes


def dequant(qweight, scales, zeros, K: int) -> np.ndarray:
    qweight = np.ascontiguousarray(qweight, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    zeros = np.ascontiguousarray(zeros, dtype=np.int32)
    N = qweight.shape[0]
    out = np.zeros((N, K), dtype=np.float64)
    lib().orc_dequant(_p(qweight), _p(scales), _p(zeros), N, K, _p(out))
    return out


def dequant_bf16(qweight, scales, zeros, K: int) -> np.ndarray:
    qweight = np.ascontiguousarray(qweight, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    zeros = np.ascontiguousarray(zeros, dtype=np.int32)
    N = qweight.shape[0]
    out = np.zeros((N, K), dtype=np.uint16)
    lib().orc_dequant_bf16(_p(qweight), _p(scales), _p(zeros), N, K, _p(out))
    return out


def linear(X: np.ndarray, qweight, scales, zeros) -> np.ndarray:
    """X bf16-bits u16 [M, K] -> Y_ref float64 [M, N] (unrounded)."""
    X = np.ascontiguousarray(X, dtype=np.uint16)
    qweight = np.ascontiguousarray(qweight, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    zeros = np.ascontiguousarray(zeros, dtype=np.int32)
    M, K = X.shape
    N = qweight.shape[0]
    Y = np.zeros((M, N), dtype=np.float64)
    lib().orc_linear(_p(X), M, K, _p(qweight), _p(scales), _p(zeros), N, _p(Y))
    return Y


def linear_sampled(X: np.ndarray, qweight, scales, zeros, m_idx, n_idx) -> np.ndarray:
    """Y_ref[i, j] for token rows m_idx[i] and output columns n_idx[j] (float64)."""
    X = np.ascontiguousarray(X, dtype=np.uint16)
    qweight = np.ascontiguousarray(qweight, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    zeros = np.ascontiguousarray(zeros, dtype=np.int32)
    m_idx = np.ascontiguousarray(np.asarray(m_idx, dtype=np.int64))
    n_idx = np.ascontiguousarray(np.asarray(n_idx, dtype=np.int64))
    M, K = X.shape
    N = qweight.shape[0]
    Y = np.zeros((m_idx.size, n_idx.size), dtype=np.float64)
    lib().orc_linear_sampled(_p(X), M, K, _p(qweight), _p(scales), _p(zeros), N, _p(m_idx), m_idx.size,
                             _p(n_idx), n_idx.size, _p(Y))
    return Y


def renorm(y_bits: np.ndarray):
    """Rows scaled to unit RMS: (bf16-bits u16 [M, N], exact float64 [M, N])."""
    y_bits = np.ascontiguousarray(y_bits, dtype=np.uint16)
    M, N = y_bits.shape
    out = np.zeros((M, N), dtype=np.uint16)
    exact = np.zeros((M, N), dtype=np.float64)
    lib().orc_renorm(_p(y_bits), M, N, _p(out), _p(exact))
    return out, exact


def awq_scale_weights(W: np.ndarray, s: np.ndarray) -> np.ndarray:
    """AWQ transform of the weights: W'[n, k] = fp32(W[n, k] * s[k])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    s = np.ascontiguousarray(s, dtype=np.float32)
    N, K = W.shape
    assert s.shape == (K,)
    out = np.empty_like(W)
    lib().orc_awq_scale_weights(_p(W), _p(s), N, K, _p(out))
    return out


def awq_scale_activations(X: np.ndarray, r: np.ndarray) -> np.ndarray:
    """AWQ transform of the activations: X'[m, k] = bf16(X[m, k] * r[k]) (bits in, bits out)."""
    X = np.ascontiguousarray(X, dtype=np.uint16)
    r = np.ascontiguousarray(r, dtype=np.float32)
    M, K = X.shape
    assert r.shape == (K,)
    out = np.empty_like(X)
    lib().orc_awq_scale_activations(_p(X), _p(r), M, K, _p(out))
    return out


def w8_quantize(W: np.ndarray, with_clipped: bool = False):
    """W float32 [N, K] -> (status, q int8 [N, K], scales bf16-bits u16 [N][, clipped u8 [N, K]]):
    symmetric INT8, one scale per output row."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    q = np.zeros((N, K), dtype=np.int8)
    sc = np.zeros(N, dtype=np.uint16)
    cl = np.zeros((N, K), dtype=np.uint8) if with_clipped else None
    st = lib().orc_w8_quantize(_p(W), N, K, _p(q), _p(sc), _p(cl) if cl is not None else None)
    return (st, q, sc, cl) if with_clipped else (st, q, sc)


def w8_linear(X: np.ndarray, q: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """X bf16 bits [M, K], q int8 [N, K], scales bf16 bits [N] -> Y float64 [M, N] (unrounded)."""
    X = np.ascontiguousarray(X, dtype=np.uint16)
    q = np.ascontiguousarray(q, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    M, K = X.shape
    N = q.shape[0]
    Y = np.empty((M, N), dtype=np.float64)
    lib().orc_w8_linear(_p(X), M, K, _p(q), _p(scales), N, _p(Y))
    return Y


def quantize_pack_g(W: np.ndarray, group: int, symmetric: bool = False, with_clipped: bool = False):
    """As quantize_pack with groups of `group` (32, 64 or 128) consecutive weights along K:
    scales and zeros [N, K/group]."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    qw = np.zeros((N, K // 8), dtype=np.uint32)
    sc = np.zeros((N, max(K // group, 1)), dtype=np.uint16)
    z = np.zeros((N, max(K // group, 1)), dtype=np.int32)
    cl = np.zeros((N, K), dtype=np.uint8) if with_clipped else None
    st = lib().orc_quantize_pack_g(_p(W), N, K, group, int(symmetric), _p(qw), _p(sc), _p(z),
                                   _p(cl) if cl is not None else None)
    return (st, qw, sc, z, cl) if with_clipped else (st, qw, sc, z)


def dequant_g(qweight, scales, zeros, K: int) -> np.ndarray:
    """W_hat float64 [N, K]; the group size is K / scales.shape[1]."""
    qweight = np.ascontiguousarray(qweight, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    zeros = np.ascontiguousarray(zeros, dtype=np.int32)
    N = qweight.shape[0]
    out = np.zeros((N, K), dtype=np.float64)
    lib().orc_dequant_g(_p(qweight), _p(scales), _p(zeros), N, K, K // scales.shape[1], _p(out))
    return out


def linear_g(X: np.ndarray, qweight, scales, zeros) -> np.ndarray:
    """Y_ref float64 [M, N] (unrounded); the group size is K / scales.shape[1]."""
    X = np.ascontiguousarray(X, dtype=np.uint16)
    qweight = np.ascontiguousarray(qweight, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    zeros = np.ascontiguousarray(zeros, dtype=np.int32)
    M, K = X.shape
    N = qweight.shape[0]
    Y = np.zeros((M, N), dtype=np.float64)
    lib().orc_linear_g(_p(X), M, K, _p(qweight), _p(scales), _p(zeros), N, K // scales.shape[1], _p(Y))
    return Y
