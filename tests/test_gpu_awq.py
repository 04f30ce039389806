"""AWQ equivalence transform on the GPU ("Axe Corsa 28B" model card, "How the
Compression Works", Stage 1; "Weight-Only Quantization and Mixed Precision",
section 3) against the oracle: w4a16_quantize_pack_awq bit-exact with the
oracle's quantisation of W diag(s), and w4a16_linear_awq -- the activation
scaling formed inside each kernel family's X preparation -- within the layer's
tolerance of the oracle product of bf16(X diag(s)^-1) and those weights.

The scales are synthetic: s_k = mean|x_k|^(1/2) over a seeded calibration batch
with salient channels, normalised to geometric mean 1 (plus power-of-two and
edge cases)."""
import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_int4_linear_b200 as w4
from synth import workloads
from tests._parity import (assert_close, bf16_dev_to_f64, bits_to_dev_bf16, dev_bf16_to_bits, dev_weights,
                           sample_rows)

pytestmark = pytest.mark.gpu

PATHS = [w4.PATH_AUTO, w4.PATH_DECODE, w4.PATH_PREFILL]


def awq_scales(K: int, seed: int):
    """(s, r = fp32(1 / s)) from a synthetic calibration batch of 64 tokens."""
    xf = oracle.bf16_to_f64(synth.activations_bf16(seed, 64, K))
    s = np.sqrt(np.abs(xf).mean(axis=0))
    s /= np.exp(np.log(s).mean())
    s = s.astype(np.float32)
    return s, (1.0 / s.astype(np.float64)).astype(np.float32)


def pack_awq(W: np.ndarray, s: np.ndarray):
    N, K = W.shape
    pw = w4.PackedWeight(N, K)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    w4.quantize_pack_awq(torch.from_numpy(np.ascontiguousarray(W)).cuda(), torch.from_numpy(s).cuda(),
                         pw.qweight, pw.scales, pw.zeros, status)
    torch.cuda.synchronize()
    pw.status = status
    return pw


def run_awq(X_bits: np.ndarray, r: np.ndarray, pw, path=w4.PATH_AUTO) -> torch.Tensor:
    M, K = X_bits.shape
    Y = torch.full((M, pw.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    nbytes = w4.workspace_bytes(M, pw.N, K)
    ws = torch.zeros(max(nbytes, 1), dtype=torch.uint8, device="cuda")
    w4.linear_awq(bits_to_dev_bf16(X_bits), torch.from_numpy(r).cuda(), pw.qweight, pw.scales, pw.zeros, Y,
                  ws if nbytes else None, path=path)
    torch.cuda.synchronize()
    return Y


@pytest.mark.parametrize("N,K", [(96, 512), (257, 1152), (640, 2048)])
def test_awq_pack_bit_exact(cuda_lib, N, K):
    W = synth.weights_f32(N + 3 * K, synth.TAG_W, N, K)
    s, _ = awq_scales(K, 41)
    pw = pack_awq(W, s)
    assert int(pw.status.item()) == 0
    st, qw, sc, z = oracle.quantize_pack(oracle.awq_scale_weights(W, s))
    assert st == oracle.OK
    np.testing.assert_array_equal(pw.qweight.cpu().numpy().view(np.uint32), qw)
    np.testing.assert_array_equal(dev_bf16_to_bits(pw.scales), sc)
    np.testing.assert_array_equal(pw.zeros.cpu().numpy(), z)


def test_awq_pack_overflow_reports_nonfinite(cuda_lib):
    W = np.full((2, 256), 1e30, dtype=np.float32)
    s = np.full(256, 1e10, dtype=np.float32)
    assert int(pack_awq(W, s).status.item()) == oracle.ERR_NONFINITE


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("M,N,K", [(1, 257, 1152), (2, 130, 1024), (3, 200, 512), (17, 384, 2048),
                                   (32, 96, 640), (70, 150, 768), (300, 320, 1024)])
def test_linear_awq_matches_oracle(cuda_lib, M, N, K, path):
    W = synth.weights_f32(M * 17 + N, synth.TAG_W, N, K)
    X = synth.activations_bf16(M + 5, M, K)
    s, r = awq_scales(K, 42)
    pw = pack_awq(W, s)
    assert int(pw.status.item()) == 0
    st, qw, sc, z = oracle.quantize_pack(oracle.awq_scale_weights(W, s))
    ref = oracle.linear(oracle.awq_scale_activations(X, r), qw, sc, z)
    assert_close(bf16_dev_to_f64(run_awq(X, r, pw, path)), ref, f"awq M={M} N={N} K={K}")


@pytest.mark.parametrize("path", PATHS)
def test_one_hot_inputs_see_the_scaled_channel(cuda_lib, path):
    """x = e_k with r_k = 2^-e_k gives Y[:, n] = w_hat'[n][k] 2^-e_k exactly: pins that the
    kernels index the inverse scales along K."""
    N, K = 96, 512
    rng = np.random.default_rng(43)
    e = rng.integers(-2, 3, size=K)
    s = np.ldexp(1.0, e).astype(np.float32)
    r = np.ldexp(1.0, -e).astype(np.float32)
    W = synth.weights_f32(44, synth.TAG_W, N, K)
    pw = pack_awq(W, s)
    st, qw, sc, z = oracle.quantize_pack(oracle.awq_scale_weights(W, s))
    ks = [0, 1, 5, 127, 128, 200, 383, 511]
    X = np.zeros((len(ks), K), dtype=np.uint16)
    for i, k in enumerate(ks):
        X[i, k] = 0x3F80
    got = bf16_dev_to_f64(run_awq(X, r, pw, path))
    wh = oracle.dequant(qw, sc, z, K)
    for i, k in enumerate(ks):
        want = oracle.bf16_to_f64(np.array([oracle.bf16_round(v * 2.0 ** -int(e[k])) for v in wh[:, k]],
                                           dtype=np.uint16))
        np.testing.assert_array_equal(got[i], want, err_msg=f"k={k}")


def test_linear_awq_equals_linear_on_prescaled_activations(cuda_lib):
    """Folding the scaling into X preparation gives the bits of scaling X first and
    calling the plain layer: both see the same BF16 X'."""
    N, K = 384, 2048
    W = synth.weights_f32(45, synth.TAG_W, N, K)
    s, r = awq_scales(K, 46)
    pw = pack_awq(W, s)
    for M, path in [(1, w4.PATH_DECODE), (2, w4.PATH_DECODE), (9, w4.PATH_DECODE), (130, w4.PATH_PREFILL)]:
        X = synth.activations_bf16(M + 47, M, K)
        Xp = oracle.awq_scale_activations(X, r)
        a = run_awq(X, r, pw, path)
        b = torch.empty_like(a)
        ws = torch.zeros(max(w4.workspace_bytes(M, N, K), 1), dtype=torch.uint8, device="cuda")
        w4.linear(bits_to_dev_bf16(Xp), pw.qweight, pw.scales, pw.zeros, b, ws, path=path)
        torch.cuda.synchronize()
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), (M, path)


@pytest.mark.parametrize("case", [c for c in workloads.decode_5120() if c.name in ("gate_up", "down")],
                         ids=lambda c: f"{c.workload}-{c.name}")
def test_linear_awq_decode_workload_sampled_rows(cuda_lib, case):
    """Full decode sizes in the benchmark's launch configuration, sampled output rows."""
    s, r = awq_scales(case.K, 48)
    W = dev_weights(case.w_seed, case.w_tag, case.N, case.K)
    pw = w4.PackedWeight(case.N, case.K)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    w4.quantize_pack_awq(W, torch.from_numpy(s).cuda(), pw.qweight, pw.scales, pw.zeros, status)
    torch.cuda.synchronize()
    del W
    assert int(status.item()) == 0
    X = synth.activations_bf16(case.x_seed, case.M, case.K)
    Y = bf16_dev_to_f64(run_awq(X, r, pw))
    rows = sample_rows(case.N, 128, case.w_seed)
    Wr = oracle.awq_scale_weights(synth.weight_rows_f32(case.w_seed, case.w_tag, case.K, rows), s)
    st, qw, sc, z = oracle.quantize_pack(Wr)
    assert st == oracle.OK
    ref = oracle.linear(oracle.awq_scale_activations(X, r), qw, sc, z)
    assert_close(Y[:, rows], ref, f"awq {case.name}")


def test_linear_awq_rejects_missing_or_misaligned_scales(cuda_lib):
    N, K = 64, 256
    pw = pack_awq(synth.weights_f32(49, synth.TAG_W, N, K), np.ones(K, dtype=np.float32))
    X = bits_to_dev_bf16(synth.activations_bf16(50, 1, K))
    Y = torch.empty((1, N), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(max(w4.workspace_bytes(1, N, K), 1), dtype=torch.uint8, device="cuda")
    lib = w4.load()
    st = lib.w4a16_linear_awq(X.data_ptr(), None, 1, K, pw.qweight.data_ptr(), pw.scales.data_ptr(),
                              pw.zeros.data_ptr(), N, Y.data_ptr(), ws.data_ptr(), ws.numel(), 0, None)
    assert st == w4.ERR_ARG
    r = torch.ones(K + 1, dtype=torch.float32, device="cuda")
    st = lib.w4a16_linear_awq(X.data_ptr(), r.data_ptr() + 4, 1, K, pw.qweight.data_ptr(), pw.scales.data_ptr(),
                              pw.zeros.data_ptr(), N, Y.data_ptr(), ws.data_ptr(), ws.numel(), 0, None)
    assert st == w4.ERR_ALIGN
