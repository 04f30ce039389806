"""W8A16 on the GPU ("Weight-Only Quantization and Mixed Precision", sections 5
and 8; "Weight-Only Quantisation", Notes) against the oracle: the per-row
symmetric INT8 quantiser and the dequantised weights bit-exact, the linear
layer within the tolerance max |Y - Y_ref| <= 2^-7 |Y_ref| + 1e-3 rms(Y_ref)
and relative Frobenius error <= 5e-3, on small shapes (every output) and the
decode workloads' full sizes (sampled output rows, the benchmark's launch
configuration)."""
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


def _quantize(W: torch.Tensor):
    pw = w4.PackedW8.from_float(W)
    torch.cuda.synchronize()
    return pw


def _linear(X_bits: np.ndarray, pw) -> torch.Tensor:
    M, K = X_bits.shape
    Y = torch.full((M, pw.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(w4.w8_workspace_bytes(M, pw.N, K), dtype=torch.uint8, device="cuda")
    w4.w8_linear(bits_to_dev_bf16(X_bits), pw.qweight, pw.scales, Y, ws)
    torch.cuda.synchronize()
    return Y


def _f32_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Nearest-even BF16 of float32 values (finite)."""
    u = np.asarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


@pytest.mark.parametrize("N,K", [(64, 128), (257, 1152), (130, 300), (8, 28672)])
def test_quantize_and_dequant_bit_exact(cuda_lib, N, K):
    W = synth.weights_f32(N * 7 + K, synth.TAG_W, N, K)
    W[0] = 0.0                      # zero row: s = 1
    W[1, :] *= np.float32(1e-30)    # tiny row
    W[2, 5] = np.float32(-3.0)      # negative extreme
    pw = _quantize(torch.from_numpy(W).cuda())
    assert int(pw.status.item()) == 0
    st, q, sc = oracle.w8_quantize(W)
    assert st == oracle.OK
    np.testing.assert_array_equal(pw.qweight.cpu().numpy(), q)
    np.testing.assert_array_equal(dev_bf16_to_bits(pw.scales), sc)
    wh = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
    w4.w8_dequant(pw.qweight, pw.scales, wh)
    torch.cuda.synchronize()
    exact = q.astype(np.float64) * oracle.bf16_to_f64(sc)[:, None]
    np.testing.assert_array_equal(dev_bf16_to_bits(wh), _f32_to_bf16_bits(exact.astype(np.float32)))


def test_quantize_reports_nonfinite(cuda_lib):
    W = torch.zeros((3, 256), dtype=torch.float32, device="cuda")
    W[1, 9] = float("inf")
    pw = _quantize(W)
    assert int(pw.status.item()) == oracle.ERR_NONFINITE


@pytest.mark.parametrize("M,N,K", [(1, 16, 128), (1, 257, 1152), (2, 130, 1024), (2, 72, 384), (3, 200, 512),
                                   (5, 96, 2048), (1, 64, 25600), (2, 640, 640)])
def test_small_shapes_all_outputs(cuda_lib, M, N, K):
    W = synth.weights_f32(M * 1000 + N + 3, synth.TAG_W, N, K)
    X = synth.activations_bf16(M + 17, M, K)
    pw = _quantize(torch.from_numpy(W).cuda())
    st, q, sc = oracle.w8_quantize(W)
    assert_close(bf16_dev_to_f64(_linear(X, pw)), oracle.w8_linear(X, q, sc), f"w8 M={M} N={N} K={K}")


def test_one_hot_inputs_pick_weight_columns(cuda_lib):
    """x = e_k gives Y[:, n] = bf16(q[n][k] s[n]) exactly: pins the byte order, the swizzled
    shared-memory reads and the row-scale addressing."""
    N, K = 200, 512
    W = synth.weights_f32(71, synth.TAG_W, N, K)
    pw = _quantize(torch.from_numpy(W).cuda())
    st, q, sc = oracle.w8_quantize(W)
    ks = [0, 1, 3, 4, 15, 16, 17, 31, 32, 100, 127, 128, 129, 255, 300, 511]
    X = np.zeros((len(ks), K), dtype=np.uint16)
    for i, k in enumerate(ks):
        X[i, k] = 0x3F80
    got = dev_bf16_to_bits(_linear(X, pw))
    exact = (q.astype(np.float64) * oracle.bf16_to_f64(sc)[:, None]).astype(np.float32)
    want = _f32_to_bf16_bits(exact)
    for i, k in enumerate(ks):
        np.testing.assert_array_equal(got[i], want[:, k], err_msg=f"k={k}")


@pytest.mark.parametrize("case", workloads.decode_5120(), ids=lambda c: f"{c.workload}-{c.name}")
def test_decode_workloads_sampled_rows(cuda_lib, case):
    W = dev_weights(case.w_seed, case.w_tag, case.N, case.K)
    pw = _quantize(W)
    del W
    assert int(pw.status.item()) == 0
    rows = sample_rows(case.N, 160, case.w_seed)
    st, q, sc = oracle.w8_quantize(synth.weight_rows_f32(case.w_seed, case.w_tag, case.K, rows))
    assert st == oracle.OK
    np.testing.assert_array_equal(pw.qweight[torch.from_numpy(rows).cuda()].cpu().numpy(), q)
    for M in (1, 2):
        X = synth.activations_bf16(case.x_seed + M, M, case.K)
        Y = bf16_dev_to_f64(_linear(X, pw))
        assert_close(Y[:, rows], oracle.w8_linear(X, q, sc), f"w8 {case.name} M={M}")
        assert np.all(np.isfinite(Y))


def test_workspace_checks_and_determinism(cuda_lib):
    N, K, M = 512, 4096, 2
    pw = _quantize(torch.from_numpy(synth.weights_f32(72, synth.TAG_W, N, K)).cuda())
    X = bits_to_dev_bf16(synth.activations_bf16(73, M, K))
    nbytes = w4.w8_workspace_bytes(M, N, K)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    Y1 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    Y2 = torch.empty_like(Y1)
    w4.w8_linear(X, pw.qweight, pw.scales, Y1, ws)
    w4.w8_linear(X, pw.qweight, pw.scales, Y2, ws)
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))
    assert int(ws[: 256 * 1024].view(torch.int32).abs().sum()) == 0  # counters left zero
    with pytest.raises(w4.W4A16Error) as e:
        w4.w8_linear(X, pw.qweight, pw.scales, Y1, ws[: nbytes - 256])
    assert e.value.status == w4.ERR_WORKSPACE
    assert w4.device_fault() == 0
