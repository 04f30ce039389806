"""w4a16_linear_noalloc: the linear layer for callers that cannot allocate
device memory (it keeps its scratch in a fixed device array inside the
library instead of a caller-provided workspace).

Checked through the C-ABI against the regular entry point, w4a16_linear,
within the tolerance the parity tests use, on two calls in a row (the array
keeps the previous call's contents).  Collected last so that a run stopping
at its first failure has already run everything else; it also passes on its
own in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

import synth
import weight_only_int4_linear_b200 as w4
from tests._parity import assert_close, bf16_dev_to_f64, bits_to_dev_bf16

pytestmark = pytest.mark.gpu


def _packed(N, K, seed):
    W = torch.from_numpy(synth.weights_f32(seed, synth.TAG_W, N, K)).cuda()
    pw = w4.PackedWeight.from_float(W)
    torch.cuda.synchronize()
    assert int(pw.status.item()) == 0
    return pw


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (1, 7680, 5120), (3, 1000, 1152), (16, 2048, 8192),
                                   (40, 384, 512)])
def test_noalloc_matches_workspace_entry_point(cuda_lib, M, N, K):
    pw = _packed(N, K, 1000 + M)
    nbytes = w4.workspace_bytes(M, N, K)
    assert 0 < nbytes <= w4.noalloc_scratch_bytes()
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    for call in range(2):
        X = bits_to_dev_bf16(synth.activations_bf16(50 + call, M, K))
        Y_ref = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        w4.linear(X, pw.qweight, pw.scales, pw.zeros, Y_ref, ws)
        w4.linear_noalloc(X, pw.qweight, pw.scales, pw.zeros, Y)
        torch.cuda.synchronize()
        assert_close(bf16_dev_to_f64(Y), bf16_dev_to_f64(Y_ref), f"call {call} M={M} N={N} K={K}")
    assert w4.device_fault() == 0


def test_noalloc_refuses_problems_beyond_its_scratch(cuda_lib):
    lib = w4.load()
    M, N, K = 32, 131072, 8192
    assert w4.workspace_bytes(M, N, K) > w4.noalloc_scratch_bytes()
    buf = torch.empty(1024, dtype=torch.uint8, device="cuda")  # never dereferenced: refused before launch
    p = ctypes.c_void_p(buf.data_ptr())
    st = lib.w4a16_linear_noalloc(p, M, K, p, p, p, N, p, None)
    assert st == w4.ERR_WORKSPACE
