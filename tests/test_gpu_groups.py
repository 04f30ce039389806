"""Quantisation groups of 32 and 64 weights on the GPU ("Quantization I: int8,
int4, the basics", Concept; "Weight-Only Quantization and Mixed Precision",
section 8) against the oracle: packing bit-exact (asymmetric and symmetric),
the linear layer within max |Y - Y_ref| <= 2^-7 |Y_ref| + 1e-3 rms(Y_ref) and
relative Frobenius <= 5e-3 on small shapes (every output), one-hot inputs
(exact BF16 of W_hat) and the decode workloads' full sizes (sampled rows)."""
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

GROUPS = [32, 64]


def _pack(W: torch.Tensor, group: int, symmetric: bool = False):
    N, K = W.shape
    pw = w4.PackedWeight(N, K, device=W.device, group=group)
    pw.status = torch.zeros(1, dtype=torch.int32, device=W.device)
    w4.quantize_pack_g(W, group, pw.qweight, pw.scales, pw.zeros, pw.status, symmetric=symmetric)
    torch.cuda.synchronize()
    return pw


def _linear(X_bits: np.ndarray, pw) -> torch.Tensor:
    M, K = X_bits.shape
    Y = torch.full((M, pw.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(max(w4.workspace_bytes_g(M, pw.N, K, pw.group), 256), dtype=torch.uint8, device="cuda")
    w4.linear_g(bits_to_dev_bf16(X_bits), pw.group, pw.qweight, pw.scales, pw.zeros, Y, ws)
    torch.cuda.synchronize()
    assert w4.device_fault() == 0
    return Y


@pytest.mark.parametrize("G", GROUPS)
@pytest.mark.parametrize("symmetric", [False, True])
def test_pack_bit_exact(cuda_lib, G, symmetric):
    N, K = 257, 1536
    W = synth.weights_f32(G + 7 * symmetric, synth.TAG_W, N, K)
    W[0] = 0.0
    W[1, :G] += np.float32(0.3)  # one one-signed group (negative zero point)
    k = np.arange(K)
    W[2] = (((k % 16) - 5) * 2.0 ** -7).astype(np.float32)
    pw = _pack(torch.from_numpy(W).cuda(), G, symmetric)
    assert int(pw.status.item()) == 0
    st, qw, sc, z = oracle.quantize_pack_g(W, G, symmetric=symmetric)
    assert st == oracle.OK
    np.testing.assert_array_equal(pw.qweight.cpu().numpy().view(np.uint32), qw)
    np.testing.assert_array_equal(dev_bf16_to_bits(pw.scales), sc)
    np.testing.assert_array_equal(pw.zeros.cpu().numpy(), z)


@pytest.mark.parametrize("G", GROUPS)
def test_pack_nonfinite_group_is_isolated(cuda_lib, G):
    """A NaN spoils only its own group: status set, that group's codes and metadata zero,
    the neighbouring groups of the same 128 weights packed as the oracle packs them."""
    N, K = 4, 256
    W = synth.weights_f32(5, synth.TAG_W, N, K)
    W[1, G + 3] = np.nan
    pw = _pack(torch.from_numpy(W).cuda(), G)
    assert int(pw.status.item()) == oracle.ERR_NONFINITE
    st, qw, sc, z = oracle.quantize_pack_g(W, G)
    assert st == oracle.ERR_NONFINITE
    np.testing.assert_array_equal(pw.qweight.cpu().numpy().view(np.uint32), qw)
    np.testing.assert_array_equal(dev_bf16_to_bits(pw.scales), sc)
    np.testing.assert_array_equal(pw.zeros.cpu().numpy(), z)


@pytest.mark.parametrize("G", GROUPS)
@pytest.mark.parametrize("M,N,K", [(1, 257, 512), (1, 640, 5120), (2, 130, 1536), (3, 96, 2048),
                                   (1, 64, 25600)])
def test_linear_small_shapes_all_outputs(cuda_lib, G, M, N, K):
    W = synth.weights_f32(M * 100 + N + G, synth.TAG_W, N, K)
    W[: N // 7] += np.float32(0.05)  # zero points spread over the grid
    X = synth.activations_bf16(M + G, M, K)
    pw = _pack(torch.from_numpy(W).cuda(), G)
    st, qw, sc, z = oracle.quantize_pack_g(W, G)
    assert_close(bf16_dev_to_f64(_linear(X, pw)), oracle.linear_g(X, qw, sc, z), f"G={G} M={M} N={N} K={K}")


@pytest.mark.parametrize("G", GROUPS)
@pytest.mark.parametrize("M", [2, 4, 9, 16, 17, 40, 70, 300, 512])
def test_batched_token_counts_all_outputs(cuda_lib, G, M):
    """Batched decode and prefill token counts: the BF16 tensor-core GEMV with one accumulator per
    quantisation group (tiles of 16 and 32 tokens, M > 32 in chunks of 32), and for groups of 64 at
    M >= 64 the GEMM with one fold per 64-K stage."""
    N, K = 200, 1024
    W = synth.weights_f32(7000 + M + G, synth.TAG_W, N, K)
    W[: N // 5] += np.float32(0.05)
    W[0, :256] += np.float32(2.0)  # one-signed groups: zero points far outside 0..15
    X = synth.activations_bf16(7100 + M, M, K)
    pw = _pack(torch.from_numpy(W).cuda(), G)
    st, qw, sc, z = oracle.quantize_pack_g(W, G)
    assert np.abs(z).max() > 128  # the fold's zero-point branch is exercised
    assert_close(bf16_dev_to_f64(_linear(X, pw)), oracle.linear_g(X, qw, sc, z), f"G={G} M={M} N={N} K={K}")


@pytest.mark.parametrize("G", GROUPS)
def test_one_hot_inputs_pick_weight_columns(cuda_lib, G):
    """x = e_k gives Y[:, n] = bf16(w_hat[n][k]) exactly: pins the sub-group split of the X
    operand, the per-lane fold and the metadata addressing of every sub-group."""
    N, K = 192, 512
    W = synth.weights_f32(60 + G, synth.TAG_W, N, K)
    W[:9] += np.float32(0.2)
    pw = _pack(torch.from_numpy(W).cuda(), G)
    st, qw, sc, z = oracle.quantize_pack_g(W, G)
    ks = [0, 1, G - 1, G, G + 7, 2 * G - 1, 127, 128, 129, 255, 256, 300, 383, 511]
    X = np.zeros((len(ks), K), dtype=np.uint16)
    for i, k in enumerate(ks):
        X[i, k] = 0x3F80
    got = dev_bf16_to_bits(_linear(X, pw))
    wh = oracle.dequant_g(qw, sc, z, K)
    for i, k in enumerate(ks):
        want = np.array([oracle.bf16_round(v) for v in wh[:, k]], dtype=np.uint16)
        np.testing.assert_array_equal(got[i], want, err_msg=f"k={k}")


@pytest.mark.parametrize("G", GROUPS)
@pytest.mark.parametrize("case", [c for c in workloads.decode_5120() if c.name in ("gate_up", "down")],
                         ids=lambda c: f"{c.workload}-{c.name}")
def test_decode_workloads_sampled_rows(cuda_lib, G, case):
    W = dev_weights(case.w_seed, case.w_tag, case.N, case.K)
    pw = _pack(W, G)
    del W
    assert int(pw.status.item()) == 0
    rows = sample_rows(case.N, 128, case.w_seed)
    st, qw, sc, z = oracle.quantize_pack_g(synth.weight_rows_f32(case.w_seed, case.w_tag, case.K, rows), G)
    assert st == oracle.OK
    np.testing.assert_array_equal(pw.qweight[torch.from_numpy(rows).cuda()].cpu().numpy().view(np.uint32), qw)
    X = synth.activations_bf16(case.x_seed, case.M, case.K)
    Y = bf16_dev_to_f64(_linear(X, pw))
    assert_close(Y[:, rows], oracle.linear_g(X, qw, sc, z), f"G={G} {case.name}")


def test_group128_through_the_group_entries_is_the_layer(cuda_lib):
    N, K, M = 320, 1024, 3
    W = torch.from_numpy(synth.weights_f32(70, synth.TAG_W, N, K)).cuda()
    a = _pack(W, 128)
    b = w4.PackedWeight.from_float(W)
    torch.cuda.synchronize()
    assert torch.equal(a.qweight, b.qweight) and torch.equal(a.zeros, b.zeros)
    X = synth.activations_bf16(71, M, K)
    Ya = _linear(X, a)
    Yb = torch.empty_like(Ya)
    ws = torch.zeros(max(w4.workspace_bytes(M, N, K), 256), dtype=torch.uint8, device="cuda")
    w4.linear(bits_to_dev_bf16(X), b.qweight, b.scales, b.zeros, Yb, ws)
    torch.cuda.synchronize()
    assert torch.equal(Ya.view(torch.int16), Yb.view(torch.int16))


def test_shape_and_group_errors(cuda_lib):
    N, K = 64, 384  # K % 512 != 0: refused for small groups
    pw = _pack(torch.from_numpy(synth.weights_f32(72, synth.TAG_W, N, K)).cuda(), 64)
    assert int(pw.status.item()) == 0
    assert w4.workspace_bytes_g(1, N, K, 64) == 0
    Y = torch.empty((1, N), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(w4.W4A16Error) as e:
        w4.linear_g(bits_to_dev_bf16(synth.activations_bf16(1, 1, K)), 64, pw.qweight, pw.scales, pw.zeros, Y, ws)
    assert e.value.status == w4.ERR_SHAPE
    lib = w4.load()
    P = pw.qweight.data_ptr()
    assert lib.w4a16_linear_g(P, 1, 512, 48, P, P, P, 16, P, P, 1 << 20, None) == w4.ERR_ARG
