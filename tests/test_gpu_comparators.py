"""The unfused W4A16 pipelines the fused kernels replace ("Quantization I: int8,
int4, the basics", Concept; "Weight-Only Quantization and Mixed Precision",
sections 1 and 7): offline dequantisation to BF16 followed by a BF16 GEMM, and
the naive three kernels (unpack, dequantise, multiply).  Both round W_hat to
BF16 before the product, which the fused kernels never do (the scale multiplies
FP32 partial sums); these tests pin the comparators' own arithmetic and record
what that rounding costs against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_int4_linear_b200 as w4
from tests._parity import assert_close, bf16_dev_to_f64, bits_to_dev_bf16

pytestmark = pytest.mark.gpu


def _packed(W):
    pw = w4.PackedWeight.from_float(torch.from_numpy(np.ascontiguousarray(W)).cuda())
    torch.cuda.synchronize()
    assert int(pw.status.item()) == 0
    return pw


@pytest.mark.parametrize("N,K", [(96, 512), (640, 2048), (257, 1152)])
def test_dequant_from_codes_matches_fused_dequant(cuda_lib, N, K):
    """unpack + dequant_codes (the naive pipeline's first two kernels) gives the bits of
    w4a16_dequant: (q - z) s is exact in FP32 and rounded once to BF16 either way."""
    pw = _packed(synth.weights_f32(N + K, synth.TAG_W, N, K))
    codes = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    a = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
    b = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
    w4.unpack(pw.qweight, K, codes)
    w4.dequant_codes(codes, pw.scales, pw.zeros, a)
    w4.dequant(pw.qweight, pw.scales, pw.zeros, K, b)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("M,N,K", [(1, 2048, 5120), (96, 384, 1152)])
def test_unfused_path_error_against_the_oracle(cuda_lib, M, N, K):
    """The unfused product X W_hat^T (W_hat in BF16, cuBLAS FP32 accumulation) stays within
    the relative Frobenius bound but exceeds the elementwise one, which the fused path meets
    on the same inputs."""
    W = synth.weights_f32(M + N + K, synth.TAG_W, N, K)
    xb = synth.activations_bf16(M + 11, M, K)
    pw = _packed(W)
    st, qw, sc, z = oracle.quantize_pack(W)
    ref = oracle.linear(xb, qw, sc, z)
    W_hat = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
    w4.dequant(pw.qweight, pw.scales, pw.zeros, K, W_hat)
    X = bits_to_dev_bf16(xb)
    Y_unfused = torch.matmul(X, W_hat.t())
    Y_fused = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(max(w4.workspace_bytes(M, N, K), 256), dtype=torch.uint8, device="cuda")
    w4.linear(X, pw.qweight, pw.scales, pw.zeros, Y_fused, ws)
    torch.cuda.synchronize()
    assert_close(bf16_dev_to_f64(Y_fused), ref, "fused")
    got = bf16_dev_to_f64(Y_unfused)
    rms = np.sqrt(np.mean(ref ** 2))
    err, bound = np.abs(got - ref), 2.0 ** -7 * np.abs(ref) + 1e-3 * rms
    rel_fro = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel_fro <= 5e-3
    assert (err > bound).any(), "the BF16 rounding of W_hat was expected to exceed the elementwise bound"
