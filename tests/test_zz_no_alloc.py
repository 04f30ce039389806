"""w4a16_linear_noalloc: the linear layer for callers that cannot allocate
device memory (it keeps its scratch in a fixed device array inside the
library instead of a caller-provided workspace).

It runs the same plan and the same kernels as w4a16_linear on the decode path,
so its outputs must equal that entry point's bit for bit, on every call of a
sequence that reuses the array with changing shapes (large N, small N, many
tokens): a stale split-K counter or partial sum left in the shared array would
change some output.  Both are also compared with the FP64 oracle under the
stated tolerance.  Collected last so that a run stopping at its first failure
has already run everything else; it also passes on its own in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_int4_linear_b200 as w4
from tests._parity import assert_close, bf16_dev_to_f64, bits_to_dev_bf16, dev_bf16_to_bits

pytestmark = pytest.mark.gpu


def _packed(N, K, seed):
    W = synth.weights_f32(seed, synth.TAG_W, N, K)
    pw = w4.PackedWeight.from_float(torch.from_numpy(W).cuda())
    torch.cuda.synchronize()
    assert int(pw.status.item()) == 0
    st, qw, sc, z = oracle.quantize_pack(W)
    assert st == oracle.OK
    return pw, (qw, sc, z)


def _regular(X, pw, path):
    M, K = X.shape
    Y = torch.full((M, pw.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    nbytes = w4.workspace_bytes(M, pw.N, K)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    w4.linear(X, pw.qweight, pw.scales, pw.zeros, Y, ws, path=path)
    return Y


# (M, N, K): one and two tokens, the tensor-core GEMV (16- and 32-token tiles), and M >= 64, where
# the no-allocation entry stays on the decode path in tiles of 32 tokens (three or more tiles reuse the
# array's counters) while w4a16_linear's automatic choice is the GEMM.
SEQUENCE = [(1, 51200, 5120), (1, 384, 512), (40, 384, 512), (2, 7680, 5120), (16, 2048, 8192),
            (100, 384, 512), (3, 1000, 1152), (130, 1000, 1152), (1, 4096, 4096)]


@pytest.mark.parametrize("repeat", [0, 1])
def test_noalloc_matches_workspace_entry_point(cuda_lib, repeat):
    """Every call bit-identical to w4a16_linear on the decode path, and within tolerance of the oracle;
    the sequence switches shapes so that each call finds the previous call's contents in the array."""
    for i, (M, N, K) in enumerate(SEQUENCE):
        pw, (qw, sc, z) = _packed(N, K, 1000 + 7 * i + M)
        Xb = synth.activations_bf16(50 + 10 * repeat + i, M, K)
        X = bits_to_dev_bf16(Xb)
        Y_dec = _regular(X, pw, w4.PATH_DECODE)
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        w4.linear_noalloc(X, pw.qweight, pw.scales, pw.zeros, Y)
        torch.cuda.synchronize()
        what = f"call {i} M={M} N={N} K={K}"
        np.testing.assert_array_equal(dev_bf16_to_bits(Y), dev_bf16_to_bits(Y_dec), err_msg=what)
        if N * K <= 8 << 20:
            assert_close(bf16_dev_to_f64(Y), oracle.linear(Xb, qw, sc, z), what)
        else:
            rows = np.unique(np.concatenate([np.arange(8), np.arange(N - 8, N), np.arange(0, N, 97)]))
            ref = oracle.linear(Xb, qw[rows], sc[rows], z[rows])
            assert_close(bf16_dev_to_f64(Y)[:, rows], ref, what)
        if M >= 64:  # the automatic choice (the GEMM) agrees within tolerance
            Y_auto = _regular(X, pw, w4.PATH_AUTO)
            torch.cuda.synchronize()
            assert_close(bf16_dev_to_f64(Y), bf16_dev_to_f64(Y_auto), what + " vs GEMM")
    assert w4.device_fault() == 0


def test_noalloc_refuses_problems_beyond_its_scratch(cuda_lib):
    lib = w4.load()
    M, N, K = 32, 131072, 8192
    assert w4.workspace_bytes(M, N, K) > w4.noalloc_scratch_bytes()
    buf = torch.empty(1024, dtype=torch.uint8, device="cuda")  # never dereferenced: refused before launch
    p = ctypes.c_void_p(buf.data_ptr())
    st = lib.w4a16_linear_noalloc(p, M, K, p, p, p, N, p, None)
    assert st == w4.ERR_WORKSPACE
