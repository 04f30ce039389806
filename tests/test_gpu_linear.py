"""GPU W4A16 linear layer against the FP64 oracle, element by element, under
the stated tolerance: max |Y - Y_ref| <= 2^-7 |Y_ref| + 1e-3 rms(Y_ref) and
relative Frobenius error <= 5e-3.

Small cases compare every output; the workloads' full sizes compare sampled
output rows (the oracle packs and multiplies just those rows, which are
independent) computed in the same launch configuration the benchmark times."""
import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_int4_linear_b200 as w4
from synth import workloads
from tests._parity import (assert_close, bf16_dev_to_f64, bits_to_dev_bf16, dev_weights, oracle_pack_rows,
                           sample_rows)

pytestmark = pytest.mark.gpu

PATHS = [w4.PATH_DECODE, w4.PATH_PREFILL]


def run_linear(X_bits: np.ndarray, pw, path=w4.PATH_AUTO) -> torch.Tensor:
    M, K = X_bits.shape
    X = bits_to_dev_bf16(X_bits)
    Y = torch.full((M, pw.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    nbytes = w4.workspace_bytes(M, pw.N, K)
    ws = torch.zeros(max(nbytes, 1), dtype=torch.uint8, device="cuda")
    w4.linear(X, pw.qweight, pw.scales, pw.zeros, Y, ws if nbytes else None, path=path)
    torch.cuda.synchronize()
    return Y


def packed_from_host(W: np.ndarray):
    pw = w4.PackedWeight.from_float(torch.from_numpy(np.ascontiguousarray(W)).cuda())
    torch.cuda.synchronize()
    assert int(pw.status.item()) == 0
    return pw


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("M,N,K", [(1, 16, 128), (1, 33, 256), (2, 130, 1024), (2, 72, 384), (3, 130, 384),
                                   (8, 256, 1024), (9, 200, 512),
                                   (16, 129, 2048), (17, 64, 640), (32, 384, 1152), (33, 100, 256),
                                   (70, 150, 768)])
def test_small_shapes_all_outputs(cuda_lib, M, N, K, path):
    W = synth.weights_f32(M * 1000 + N, synth.TAG_W, N, K)
    X = synth.activations_bf16(M + 7, M, K)
    pw = packed_from_host(W)
    st, qw, sc, z = oracle.quantize_pack(W)
    Y = run_linear(X, pw, path)
    assert_close(bf16_dev_to_f64(Y), oracle.linear(X, qw, sc, z), f"M={M} N={N} K={K}")


@pytest.mark.parametrize("M", [3, 4, 5, 7, 8, 9, 12, 15, 16, 17, 20, 24, 31, 33, 48, 63])
def test_small_batch_token_counts_all_outputs(cuda_lib, M):
    """Every token count of the 3-16-token integer GEMV (tiles of 4, 8 and 16 tokens; M > 16 in chunks of
    16 with a smaller last tile), K / 128 a multiple of 8, ragged N."""
    N, K = 200, 1024
    W = synth.weights_f32(3000 + M, synth.TAG_W, N, K)
    X = synth.activations_bf16(3100 + M, M, K)
    pw = packed_from_host(W)
    st, qw, sc, z = oracle.quantize_pack(W)
    Y = run_linear(X, pw, w4.PATH_DECODE)
    assert_close(bf16_dev_to_f64(Y), oracle.linear(X, qw, sc, z), f"M={M} N={N} K={K}")
    assert w4.device_fault() == 0


@pytest.mark.parametrize("path", PATHS)
def test_one_hot_inputs_pick_weight_columns(cuda_lib, path):
    """x = e_k must give Y[:, n] = bf16(w_hat[n][k]) exactly: pins nibble order,
    group indexing and scale/zero addressing through the GPU path."""
    N, K = 96, 512
    W = synth.weights_f32(5, synth.TAG_W, N, K)
    W[:9] += np.float32(0.25)  # negative zero points on some rows
    pw = packed_from_host(W)
    st, qw, sc, z = oracle.quantize_pack(W)
    ks = [0, 1, 4, 7, 8, 15, 16, 31, 127, 128, 129, 255, 300, 511]
    X = np.zeros((len(ks), K), dtype=np.uint16)
    for i, k in enumerate(ks):
        X[i, k] = 0x3F80
    Y = run_linear(X, pw, path)
    wh_bits = oracle.dequant_bf16(qw, sc, z, K)
    got = Y.view(torch.int16).cpu().numpy().view(np.uint16)
    for i, k in enumerate(ks):
        np.testing.assert_array_equal(got[i], wh_bits[:, k], err_msg=f"k={k}")


def test_constant_inputs(cuda_lib):
    """A constant row restricted to one group sums that group's w_hat."""
    N, K = 64, 384
    W = synth.weights_f32(6, synth.TAG_W, N, K)
    pw = packed_from_host(W)
    st, qw, sc, z = oracle.quantize_pack(W)
    X = np.zeros((2, K), dtype=np.uint16)
    X[0, 128:256] = 0x4000  # 2.0
    X[1, :] = 0xBF80        # -1.0
    Y = bf16_dev_to_f64(run_linear(X, pw))
    wh = oracle.dequant(qw, sc, z, K)
    assert_close(Y, np.stack([2.0 * wh[:, 128:256].sum(1), -wh.sum(1)]), "constant rows")


def test_single_gemv_full(cuda_lib):
    case = workloads.single_gemv()[0]
    pw = packed_from_host(synth.weights_f32(case.w_seed, case.w_tag, case.N, case.K))
    X = synth.activations_bf16(case.x_seed, case.M, case.K)
    st, qw, sc, z = oracle.quantize_pack(synth.weights_f32(case.w_seed, case.w_tag, case.N, case.K))
    Y = run_linear(X, pw)
    stats = assert_close(bf16_dev_to_f64(Y), oracle.linear(X, qw, sc, z), case.name)
    # the final BF16 rounding of Y alone contributes ~1.7e-3 relative Frobenius error
    assert stats["rel_fro"] < 2.5e-3


def _device_packed(case):
    W = dev_weights(case.w_seed, case.w_tag, case.N, case.K)
    pw = w4.PackedWeight.from_float(W)
    torch.cuda.synchronize()
    del W
    assert int(pw.status.item()) == 0
    return pw


@pytest.mark.parametrize("case", workloads.decode_5120() + workloads.small_batch_8192(),
                         ids=lambda c: f"{c.workload}-{c.name}")
def test_decode_workloads_sampled_rows(cuda_lib, case):
    pw = _device_packed(case)
    X = synth.activations_bf16(case.x_seed, case.M, case.K)
    Y = run_linear(X, pw)
    rows = sample_rows(case.N, 192, case.w_seed)
    qw, sc, z = oracle_pack_rows(case, rows)
    ref = oracle.linear(X, qw, sc, z)  # [M, len(rows)]
    got = bf16_dev_to_f64(Y)[:, rows]
    assert_close(got, ref, f"{case.workload}/{case.name}")
    assert np.all(np.isfinite(bf16_dev_to_f64(Y)))


@pytest.mark.parametrize("case", workloads.prefill_8192(), ids=lambda c: f"{c.workload}-{c.name}")
def test_prefill_workloads_sampled(cuda_lib, case):
    pw = _device_packed(case)
    X = synth.activations_bf16(case.x_seed, case.M, case.K)
    Y = bf16_dev_to_f64(run_linear(X, pw))
    rows = sample_rows(case.N, 64, case.w_seed)
    qw, sc, z = oracle_pack_rows(case, rows)
    m_idx = sample_rows(case.M, 48, case.x_seed)
    ref = oracle.linear_sampled(X, qw, sc, z, m_idx, np.arange(rows.size))
    assert_close(Y[np.ix_(m_idx, rows)], ref, f"{case.workload}/{case.name}")


def test_workspace_reuse_and_errors(cuda_lib):
    N, K, M = 512, 4096, 1
    W = synth.weights_f32(9, synth.TAG_W, N, K)
    pw = packed_from_host(W)
    X = bits_to_dev_bf16(synth.activations_bf16(9, M, K))
    nbytes = w4.workspace_bytes(M, N, K)
    assert nbytes > 0  # small N splits K across CTAs
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    Y1 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    Y2 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    w4.linear(X, pw.qweight, pw.scales, pw.zeros, Y1, ws)
    w4.linear(X, pw.qweight, pw.scales, pw.zeros, Y2, ws)
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))  # deterministic split-K order
    with pytest.raises(w4.W4A16Error) as e:  # not even the 256 KB counter area
        w4.linear(X, pw.qweight, pw.scales, pw.zeros, Y1, ws[: 128 * 1024])
    assert e.value.status == w4.ERR_WORKSPACE
    with pytest.raises(w4.W4A16Error) as e:
        w4.linear(X, pw.qweight, pw.scales, pw.zeros, Y1, None)
    assert e.value.status == w4.ERR_WORKSPACE


def test_one_workspace_shared_by_shapes_and_paths(cuda_lib):
    """Calls of different shapes and paths, ordered on one stream, share one
    workspace initialised once: each call must leave the split-K counters the
    next one relies on at zero, whatever it writes elsewhere."""
    shapes = [(1, 384, 8192), (1, 256, 28672), (3, 384, 8192), (70, 256, 1024), (1, 384, 8192), (1, 256, 28672),
              (17, 640, 2048), (1, 384, 8192)]
    packed, inputs, refs = {}, {}, {}
    for M, N, K in shapes:
        if (N, K) not in packed:
            W = synth.weights_f32(N + K, synth.TAG_W, N, K)
            packed[(N, K)] = (packed_from_host(W), oracle.quantize_pack(W)[1:])
        if (M, N, K) not in inputs:
            inputs[(M, N, K)] = synth.activations_bf16(M + K, M, K)
            qw, sc, z = packed[(N, K)][1]
            refs[(M, N, K)] = oracle.linear(inputs[(M, N, K)], qw, sc, z)
    nbytes = max(w4.workspace_bytes(M, N, K) for M, N, K in shapes)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    w4.workspace_init(ws)
    outs = []
    for M, N, K in shapes:
        pw = packed[(N, K)][0]
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        w4.linear(bits_to_dev_bf16(inputs[(M, N, K)]), pw.qweight, pw.scales, pw.zeros, Y, ws)
        outs.append(Y)
    torch.cuda.synchronize()
    for (M, N, K), Y in zip(shapes, outs):
        assert_close(bf16_dev_to_f64(Y), refs[(M, N, K)], f"shared workspace M={M} N={N} K={K}")
    assert w4.device_fault() == 0


@pytest.mark.parametrize("N", [28672, 1001])  # the wide kernel (N % 8 == 0, values in registers) and the general one
def test_renorm_rows(cuda_lib, N):
    rng = np.random.default_rng(4)
    y = torch.from_numpy(rng.standard_normal((3, N)).astype(np.float32) * 5).to(torch.bfloat16).cuda()
    y[2].zero_()
    out = torch.empty_like(y)
    w4.renorm_rows(y, out)
    torch.cuda.synchronize()
    ref_bits, exact = oracle.renorm(y.view(torch.int16).cpu().numpy().view(np.uint16))
    got = out.view(torch.int16).cpu().numpy().view(np.uint16).astype(np.int32)
    # FP32 sum of squares vs FP64: at most one BF16 ulp apart, almost always equal
    assert np.max(np.abs(got - ref_bits.astype(np.int32))) <= 1
    assert np.mean(got != ref_bits) < 1e-3


def _groups_with_zero_points(N, K, zs, seed):
    """Weights whose group g of row n has scale 1/16 and zero point
    zs[(n + g) % len(zs)]: the group is rescaled onto [lo, lo + 15/16] with
    lo = -z/16, so (hi - lo)/15 = 1/16 exactly and z = rint(-lo/s)."""
    W = synth.weights_f32(seed, synth.TAG_W, N, K).astype(np.float64).reshape(N, K // 128, 128)
    lo_w = W.min(axis=2, keepdims=True)
    hi_w = W.max(axis=2, keepdims=True)
    z = np.array([[zs[(n + g) % len(zs)] for g in range(K // 128)] for n in range(N)], dtype=np.float64)
    lo = (-z / 16.0)[:, :, None]
    W = lo + (W - lo_w) / (hi_w - lo_w) * (15.0 / 16.0)
    return W.reshape(N, K).astype(np.float32), z.astype(np.int64)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("M", [1, 8, 70])
def test_zero_points_far_outside_the_code_range(cuda_lib, M, path):
    """One-signed groups have zero points far from 0..15 (here up to +-2000):
    the kernels take a different branch for |z| > 128; both sides of that
    boundary, and z = +-128 on it, must match the oracle."""
    zs = [0, 7, 15, 127, 128, 129, -127, -128, -129, 300, -300, 2000, -2000, 64]
    N, K = 130, 1024
    W, z_expect = _groups_with_zero_points(N, K, zs, 77)
    st, qw, sc, z = oracle.quantize_pack(W)
    assert st == oracle.OK
    np.testing.assert_array_equal(z, z_expect)
    pw = packed_from_host(W)
    assert torch.equal(pw.zeros.cpu(), torch.from_numpy(z.astype(np.int32)))
    X = synth.activations_bf16(900 + M, M, K)
    Y = run_linear(X, pw, path)
    assert_close(bf16_dev_to_f64(Y), oracle.linear(X, qw, sc, z), f"M={M}")


def test_host_buffer_entry_chained_through_host(cuda_lib):
    """Two one-token layers through w4a16_linear_host, the second reading the first's host output: the
    transfers are kernels of the launch chain (mapped host buffers), so the second call's copy must wait for
    the first call's stores into host memory.  Same bits as the device-buffer chain."""
    K1, N1, N2 = 2048, 3072, 1000  # layer 2: K = 3072
    W1 = synth.weights_f32(31, synth.TAG_W, N1, K1)
    W2 = synth.weights_f32(32, synth.TAG_W, N2, N1)
    p1, p2 = packed_from_host(W1), packed_from_host(W2)
    xb = synth.activations_bf16(33, 1, K1)
    Y1_ref = run_linear(xb, p1)
    Y2_ref = run_linear(Y1_ref.view(torch.int16).cpu().numpy().view(np.uint16), p2)
    X_host = torch.from_numpy(xb.view(np.int16)).pin_memory()
    H_host = torch.full((1, N1), -1, dtype=torch.int16).pin_memory()
    Y_host = torch.full((1, N2), -1, dtype=torch.int16).pin_memory()
    X1 = torch.empty((1, K1), dtype=torch.bfloat16, device="cuda")
    Y1 = torch.empty((1, N1), dtype=torch.bfloat16, device="cuda")
    X2 = torch.empty((1, N1), dtype=torch.bfloat16, device="cuda")
    Y2 = torch.empty((1, N2), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(max(w4.workspace_bytes(1, N1, K1), w4.workspace_bytes(1, N2, N1)), dtype=torch.uint8,
                     device="cuda")
    for _ in range(3):
        H_host.fill_(-1)
        Y_host.fill_(-1)
        w4.linear_host(X_host, X1, p1.qweight, p1.scales, p1.zeros, Y1, H_host, ws)
        w4.linear_host(H_host, X2, p2.qweight, p2.scales, p2.zeros, Y2, Y_host, ws)
        torch.cuda.synchronize()
        assert torch.equal(H_host, Y1_ref.view(torch.int16).cpu())
        assert torch.equal(Y_host, Y2_ref.view(torch.int16).cpu())
        assert torch.equal(Y2.view(torch.int16), Y2_ref.view(torch.int16))


@pytest.mark.parametrize("M,N,K", [(1, 640, 1024), (2, 256, 2048), (96, 384, 1152)])
def test_host_buffer_entry_matches_device_entry(cuda_lib, M, N, K):
    """w4a16_linear_host (copies in and out on the stream) gives the same bits as w4a16_linear."""
    W = synth.weights_f32(M + N + K, synth.TAG_W, N, K)
    pw = packed_from_host(W)
    xb = synth.activations_bf16(M + 3, M, K)
    Y_ref = run_linear(xb, pw)
    X_host = torch.from_numpy(xb.view(np.int16)).pin_memory()
    Y_host = torch.full((M, N), -1, dtype=torch.int16).pin_memory()
    X_dev = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    Y_dev = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(max(w4.workspace_bytes(M, N, K), 1), dtype=torch.uint8, device="cuda")
    w4.linear_host(X_host, X_dev, pw.qweight, pw.scales, pw.zeros, Y_dev, Y_host, ws)
    torch.cuda.synchronize()
    assert torch.equal(Y_host, Y_ref.view(torch.int16).cpu())
