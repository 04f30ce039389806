"""GPU quantise/pack, unpack and dequant against the oracle: bit-exact.

The weights are drawn on the device by the same counter-based generator the
host uses (checked bit-exact first), so the oracle sees identical inputs."""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import workloads
from tests._parity import dev_bf16_to_bits, dev_weights, oracle_pack_rows, sample_rows

pytestmark = pytest.mark.gpu


def test_device_generator_matches_host(cuda_lib):
    for (seed, tag, N, K) in [(0, synth.TAG_W, 64, 4096), (3, synth.TAG_W_STACK + 2, 33, 256)]:
        Wd = dev_weights(seed, tag, N, K).cpu().numpy()
        Wh = synth.weights_f32(seed, tag, N, K)
        np.testing.assert_array_equal(Wd.view(np.uint32), Wh.view(np.uint32))
    # far into a large tensor: offsets past 2^31 elements
    rows = np.array([0, 57343], dtype=np.int64)
    K = 8192
    out = torch.empty((2, K), dtype=torch.float32, device="cuda")
    for i, r in enumerate(rows):
        synth.fill_weights_device(7, synth.TAG_W, out[i].data_ptr(), K, offset=int(r) * K)
    np.testing.assert_array_equal(out.cpu().numpy().view(np.uint32),
                                  synth.weight_rows_f32(7, synth.TAG_W, K, rows).view(np.uint32))


def _pack_dev(W: torch.Tensor):
    pw = cuda_pack(W)
    torch.cuda.synchronize()
    return pw


def cuda_pack(W):
    import weight_only_int4_linear_b200 as w4
    return w4.PackedWeight.from_float(W)


def _check_packed_rows(pw, rows, qw, sc, z):
    idx = torch.from_numpy(rows).cuda()
    np.testing.assert_array_equal(pw.qweight[idx].cpu().numpy().view(np.uint32), qw)
    np.testing.assert_array_equal(dev_bf16_to_bits(pw.scales[idx]), sc)
    np.testing.assert_array_equal(pw.zeros[idx].cpu().numpy(), z)


@pytest.mark.parametrize("case", workloads.single_gemv() + workloads.decode_5120()[:2],
                         ids=lambda c: f"{c.workload}-{c.name}")
def test_pack_bit_exact_full(cuda_lib, case):
    W = dev_weights(case.w_seed, case.w_tag, case.N, case.K)
    pw = _pack_dev(W)
    assert int(pw.status.item()) == 0
    st, qw, sc, z = oracle.quantize_pack(synth.weights_f32(case.w_seed, case.w_tag, case.N, case.K))
    assert st == oracle.OK
    np.testing.assert_array_equal(pw.qweight.cpu().numpy().view(np.uint32), qw)
    np.testing.assert_array_equal(dev_bf16_to_bits(pw.scales), sc)
    np.testing.assert_array_equal(pw.zeros.cpu().numpy(), z)


@pytest.mark.parametrize("case", workloads.decode_5120()[2:] + workloads.prefill_8192(ms=[512]),
                         ids=lambda c: f"{c.workload}-{c.name}")
def test_pack_bit_exact_sampled_rows(cuda_lib, case):
    W = dev_weights(case.w_seed, case.w_tag, case.N, case.K)
    pw = _pack_dev(W)
    del W
    assert int(pw.status.item()) == 0
    rows = sample_rows(case.N, 256, case.w_seed)
    _check_packed_rows(pw, rows, *oracle_pack_rows(case, rows))


def test_pack_edge_groups(cuda_lib):
    """Hand-worked groups, shifted/scaled groups (negative and large zero points,
    tiny and huge ranges, constant and zero groups) and a ragged row count."""
    rng = np.random.default_rng(0)
    N, K = 37, 384
    W = synth.weights_f32(11, synth.TAG_W, N, K).reshape(-1, 128)
    shift = rng.choice([0.0, 2.5, -10.0, 10.0], size=(W.shape[0], 1)).astype(np.float32)
    scale = rng.choice([1.0, 1e-3, 40.0, 1e-30, 1e30], size=(W.shape[0], 1)).astype(np.float32)
    W = ((W + shift * np.float32(0.02)) * scale).astype(np.float32)
    k = np.arange(128)
    W[0] = ((k % 16) - 5) * 2.0 ** -7
    W[1] = 0.3
    W[2] = 0.0
    W[3] = np.where(k == 0, -4.5, np.where(k == 1, 10.5, (k % 12) - 4)) * 2.0 ** -7
    W[4] = 1e-40  # subnormal binary32 constant group
    W[5, :64] = 3e-39
    W[5, 64:] = -2e-39
    W = W.reshape(N, K)
    pw = _pack_dev(torch.from_numpy(W).cuda())
    assert int(pw.status.item()) == 0
    st, qw, sc, z = oracle.quantize_pack(W)
    assert st == oracle.OK
    np.testing.assert_array_equal(pw.qweight.cpu().numpy().view(np.uint32), qw)
    np.testing.assert_array_equal(dev_bf16_to_bits(pw.scales), sc)
    np.testing.assert_array_equal(pw.zeros.cpu().numpy(), z)


def test_pack_reports_nonfinite(cuda_lib):
    W = torch.zeros((4, 256), dtype=torch.float32, device="cuda")
    W[2, 130] = float("inf")
    pw = _pack_dev(W)
    assert int(pw.status.item()) == oracle.ERR_NONFINITE
    # a clean call clears the status word again
    pw2 = _pack_dev(torch.zeros((4, 256), dtype=torch.float32, device="cuda"))
    assert int(pw2.status.item()) == 0


def test_unpack_and_dequant_bit_exact(cuda_lib):
    import weight_only_int4_linear_b200 as w4
    N, K = 300, 1024
    W = synth.weights_f32(21, synth.TAG_W, N, K)
    W[:7] += np.float32(0.3)  # negative zero points
    pw = _pack_dev(torch.from_numpy(W).cuda())
    st, qw, sc, z = oracle.quantize_pack(W)
    codes = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    w4.unpack(pw.qweight, K, codes)
    wh = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
    w4.dequant(pw.qweight, pw.scales, pw.zeros, K, wh)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(codes.cpu().numpy(), oracle.unpack(qw, K))
    np.testing.assert_array_equal(dev_bf16_to_bits(wh), oracle.dequant_bf16(qw, sc, z, K))
    # integer (q - z) values, bit-exact
    qz_gpu = codes.cpu().numpy().astype(np.int64) - np.repeat(pw.zeros.cpu().numpy(), 128, axis=1)
    qz_ref = oracle.unpack(qw, K).astype(np.int64) - np.repeat(z, 128, axis=1)
    np.testing.assert_array_equal(qz_gpu, qz_ref)
