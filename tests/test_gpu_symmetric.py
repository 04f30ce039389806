"""Symmetric INT4 ("Quantization I: int8, int4, the basics", Concept: a scale
and no zero point) on the GPU: w4a16_quantize_pack_sym against the oracle,
bit-exact, and the unchanged linear kernels on symmetric-packed weights (signed
code q stored as q + 8 with zero point 8) against the oracle product."""
import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_int4_linear_b200 as w4
from synth import workloads
from tests._parity import assert_close, bf16_dev_to_f64, dev_bf16_to_bits, dev_weights
from tests.test_gpu_linear import run_linear

pytestmark = pytest.mark.gpu


def _pack_sym(W: torch.Tensor):
    pw = w4.PackedWeight.from_float(W, symmetric=True)
    torch.cuda.synchronize()
    return pw


def _assert_packed_equal(pw, qw, sc, z):
    np.testing.assert_array_equal(pw.qweight.cpu().numpy().view(np.uint32), qw)
    np.testing.assert_array_equal(dev_bf16_to_bits(pw.scales), sc)
    np.testing.assert_array_equal(pw.zeros.cpu().numpy(), z)


@pytest.mark.parametrize("case", workloads.single_gemv()[:1] + workloads.decode_5120()[:2],
                         ids=lambda c: f"{c.workload}-{c.name}")
def test_sym_pack_bit_exact(cuda_lib, case):
    W = dev_weights(case.w_seed, case.w_tag, case.N, case.K)
    pw = _pack_sym(W)
    assert int(pw.status.item()) == 0
    st, qw, sc, z = oracle.quantize_pack(synth.weights_f32(case.w_seed, case.w_tag, case.N, case.K),
                                         symmetric=True)
    assert st == oracle.OK
    _assert_packed_equal(pw, qw, sc, z)
    assert int(pw.zeros.min()) == 8 and int(pw.zeros.max()) == 8


def test_sym_pack_edge_groups(cuda_lib):
    """Hand-worked grid and tie groups, negative extremes, zero, subnormal, tiny and huge groups."""
    rng = np.random.default_rng(1)
    N, K = 29, 384
    W = synth.weights_f32(12, synth.TAG_W, N, K).reshape(-1, 128)
    scale = rng.choice([1.0, 1e-3, 40.0, 1e-30, 1e30], size=(W.shape[0], 1)).astype(np.float32)
    W = (W * scale).astype(np.float32)
    k = np.arange(128)
    S7 = 2.0 ** -7
    W[0] = ((k % 15) - 7) * S7
    W[1] = 0.0
    W[1, :6] = np.array([7.0, 2.5, -3.5, -0.5, 6.5, -6.5]) * S7
    W[2] = 0.0
    W[3] = -0.01
    W[3, 9] = -7 * S7
    W[4] = 1e-40
    W[5, :64] = 3e-39
    W[5, 64:] = -2e-39
    W = W.reshape(N, K)
    pw = _pack_sym(torch.from_numpy(W).cuda())
    assert int(pw.status.item()) == 0
    st, qw, sc, z = oracle.quantize_pack(W, symmetric=True)
    assert st == oracle.OK
    _assert_packed_equal(pw, qw, sc, z)


def test_sym_pack_reports_nonfinite(cuda_lib):
    W = torch.zeros((4, 256), dtype=torch.float32, device="cuda")
    W[1, 3] = float("nan")
    assert int(_pack_sym(W).status.item()) == oracle.ERR_NONFINITE


@pytest.mark.parametrize("path", [w4.PATH_AUTO, w4.PATH_DECODE, w4.PATH_PREFILL])
@pytest.mark.parametrize("M,N,K", [(1, 257, 1152), (2, 130, 1024), (5, 384, 2048), (32, 200, 512),
                                   (300, 320, 1024)])
def test_linear_on_symmetric_weights(cuda_lib, M, N, K, path):
    W = synth.weights_f32(M * 131 + N, synth.TAG_W, N, K)
    X = synth.activations_bf16(M + 3, M, K)
    pw = _pack_sym(torch.from_numpy(W).cuda())
    assert int(pw.status.item()) == 0
    st, qw, sc, z = oracle.quantize_pack(W, symmetric=True)
    Y = run_linear(X, pw, path)
    assert_close(bf16_dev_to_f64(Y), oracle.linear(X, qw, sc, z), f"sym M={M} N={N} K={K}")


def test_symmetric_error_against_unquantised_weights(cuda_lib):
    """Both formats keep every weight within half a step of its own grid, and the
    symmetric step max|w| / 7 lies between 15/14 and 15/7 times the affine step
    (hi - lo) / 15, so the symmetric reconstruction error is larger, by at most
    about that factor."""
    N, K = 256, 1024
    W = synth.weights_f32(77, synth.TAG_W, N, K)
    wh = {}
    for sym in (False, True):
        pw = w4.PackedWeight.from_float(torch.from_numpy(W).cuda(), symmetric=sym)
        out = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
        w4.dequant(pw.qweight, pw.scales, pw.zeros, K, out)
        torch.cuda.synchronize()
        wh[sym] = bf16_dev_to_f64(out)
    e_aff = np.linalg.norm(wh[False] - W) / np.linalg.norm(W)
    e_sym = np.linalg.norm(wh[True] - W) / np.linalg.norm(W)
    assert e_aff < e_sym < 2.5 * e_aff
