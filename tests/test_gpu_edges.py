"""Activations with extreme per-group dynamic range through every kernel family,
against the FP64 oracle under the stated tolerance, one token row at a time.

The decode kernels write each group of 128 activations as the integer
x * 2^(21 - E) in three signed base-256 digits (E the exponent of the group's
largest magnitude): exact for values within 2^14 of that maximum, rounded at
2^(E - 21) below it.  The activations themselves are never quantised ("Axe
Corsa 28B" model card, "How the Compression Works": activations stay BF16), so
this rounding must stay inside the tolerance whatever the group holds: values
twenty binades below the group maximum, exact and signed zeros, all-zero
groups and rows, negative maxima, BF16 subnormals, the smallest normal
binades, magnitudes near 2^100 and the largest finite BF16.

Each row is compared against its own oracle row (the tolerance's rms taken over
that row), so a row of tiny values is held to a bound of its own size.  Rows of
subnormal activations times ordinary weights give outputs below the smallest
normal BF16, where the output's own spacing (2^-133) is coarser than the
relative bound; there the tolerance's absolute term of half that spacing
decides, and a separate case scales the weights by 2^20 so that subnormal
inputs give normal outputs, held to the relative bound alone."""
import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_int4_linear_b200 as w4
from synth import edge
from tests._parity import assert_close, bf16_dev_to_f64, bits_to_dev_bf16

pytestmark = pytest.mark.gpu

ALL = list(edge.KINDS)
# The kernels on BF16 operands -- the GEMM, and the tensor-core GEMV for groups of 32/64 beyond one
# token -- multiply BF16 (q - c) by BF16 x and sum in FP32 before the scale: activations must stay below
# 2^113 in magnitude, so the largest finite BF16 is outside their range (the integer GEMVs take every
# finite BF16 value).
PREFILL_KINDS = [k for k in ALL if k != "max_finite"]
BF16_KINDS = PREFILL_KINDS
# x * inv_s of the largest finite BF16 overflows for inv_s > 1: the transformed activation is not finite.
AWQ_KINDS = [k for k in ALL if k != "max_finite"]


def _pack(N, K, seed, group=128, w_scale=1.0):
    W = synth.weights_f32(seed, synth.TAG_W, N, K) * np.float32(w_scale)
    W[: min(3, N), :K // 2] += np.float32(0.3)  # a few one-signed groups: zero points outside 0..15
    Wd = torch.from_numpy(np.ascontiguousarray(W)).cuda()
    if group == 128:
        pw = w4.PackedWeight.from_float(Wd)
        st, qw, sc, z = oracle.quantize_pack(W)
    else:
        pw = w4.PackedWeight(N, K, group=group)
        pw.status = torch.zeros(1, dtype=torch.int32, device="cuda")
        w4.quantize_pack_g(Wd, group, pw.qweight, pw.scales, pw.zeros, pw.status)
        st, qw, sc, z = oracle.quantize_pack_g(W, group)
    torch.cuda.synchronize()
    assert int(pw.status.item()) == 0 and st == oracle.OK
    return pw, (qw, sc, z)


def _check_rows(Y: torch.Tensor, Y_ref: np.ndarray, kinds, what: str):
    got = bf16_dev_to_f64(Y)
    for m, kind in enumerate(kinds):
        assert_close(got[m], Y_ref[m], f"{what} row {m} ({kind})")


def _linear(X_bits, pw, path):
    M, K = X_bits.shape
    Y = torch.full((M, pw.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    nbytes = w4.workspace_bytes(M, pw.N, K)
    ws = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device="cuda")
    w4.linear(bits_to_dev_bf16(X_bits), pw.qweight, pw.scales, pw.zeros, Y, ws, path=path)
    torch.cuda.synchronize()
    assert w4.device_fault() == 0
    return Y


@pytest.mark.parametrize("N,K", [(200, 1024), (136, 5120)])
@pytest.mark.parametrize("kind", ALL)
def test_one_token(cuda_lib, N, K, kind):
    """M = 1: the integer GEMV for one token (X digits formed inside the kernel)."""
    pw, (qw, sc, z) = _pack(N, K, 11)
    X = edge.activations_bf16(101 + ALL.index(kind), [kind], K)
    Y = _linear(X, pw, w4.PATH_AUTO)
    _check_rows(Y, oracle.linear(X, qw, sc, z), [kind], f"M=1 N={N} K={K}")


@pytest.mark.parametrize("M", [1, 2, 5, 40, 70])
def test_subnormal_inputs_normal_outputs(cuda_lib, M):
    """Subnormal activations against weights of magnitude ~2^14: outputs in the normal range, so the
    relative bound applies in full; every kernel family (M = 70 is the GEMM)."""
    N, K = 200, 2048
    kinds = ["subnormal" if m % 2 == 0 else "subnormal_mixed" for m in range(M)]
    pw, (qw, sc, z) = _pack(N, K, 18, w_scale=2.0 ** 20)
    X = edge.activations_bf16(800 + M, kinds, K)
    Y = _linear(X, pw, w4.PATH_AUTO)
    Y_ref = oracle.linear(X, qw, sc, z)
    assert np.abs(Y_ref[0]).max() > 2.0 ** -120  # outputs in the normal BF16 range
    _check_rows(Y, Y_ref, kinds, f"subnormal x large weights M={M}")


@pytest.mark.parametrize("pair", [(ALL[i], ALL[(i + 1) % len(ALL)]) for i in range(len(ALL))])
def test_two_tokens(cuda_lib, pair):
    """M = 2: the integer GEMV for two tokens."""
    N, K = 200, 2048
    pw, (qw, sc, z) = _pack(N, K, 12)
    X = edge.activations_bf16(202, list(pair), K)
    Y = _linear(X, pw, w4.PATH_AUTO)
    _check_rows(Y, oracle.linear(X, qw, sc, z), pair, "M=2")


@pytest.mark.parametrize("M", [3, 5, 8, 12, 16])
def test_small_batch_integer_gemv(cuda_lib, M):
    """2 <= M <= 16: digit planes prepared once per launch (4-, 8- and 16-token tiles), mma.sync u8 x s8."""
    N, K = 200, 2048
    kinds = [ALL[m % len(ALL)] for m in range(M)]
    pw, (qw, sc, z) = _pack(N, K, 13)
    X = edge.activations_bf16(300 + M, kinds, K)
    Y = _linear(X, pw, w4.PATH_DECODE)
    _check_rows(Y, oracle.linear(X, qw, sc, z), kinds, f"M={M}")


@pytest.mark.parametrize("M,K", [(9, 640), (16, 640), (17, 2048), (40, 2048)])
def test_tensor_core_gemv(cuda_lib, M, K):
    """The codes as 8-bit A operands in tensor memory against the digit planes of every token, tcgen05
    kind::i8 (16- and 32-token tiles): 17 or more tokens, or any count when K / 128 is not a multiple of 8
    (M = 40 runs a 32-token and an 8-token launch)."""
    N = 200
    kinds = [ALL[m % len(ALL)] for m in range(M)]
    pw, (qw, sc, z) = _pack(N, K, 13)
    X = edge.activations_bf16(300 + M, kinds, K)
    Y = _linear(X, pw, w4.PATH_DECODE)
    _check_rows(Y, oracle.linear(X, qw, sc, z), kinds, f"M={M} K={K}")


@pytest.mark.parametrize("group", [32, 64])
@pytest.mark.parametrize("batched", [False, True])
def test_small_groups(cuda_lib, group, batched):
    """Groups of 32 and 64: one token per call on the integer GEMV with per-sub-group digit rows (every
    kind), or all rows in one call on the BF16 tensor-core GEMV (every kind but the largest finite)."""
    N, K = 200, 1024
    kinds = BF16_KINDS if batched else ALL
    pw, (qw, sc, z) = _pack(N, K, 14, group)
    X = edge.activations_bf16(400 + group, kinds, K)
    M = len(kinds)
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(max(w4.workspace_bytes_g(M, N, K, group), 256), dtype=torch.uint8, device="cuda")
    if batched:
        w4.linear_g(bits_to_dev_bf16(X), group, pw.qweight, pw.scales, pw.zeros, Y, ws)
    else:
        for m in range(M):
            w4.linear_g(bits_to_dev_bf16(X[m:m + 1]), group, pw.qweight, pw.scales, pw.zeros, Y[m:m + 1], ws)
    torch.cuda.synchronize()
    assert w4.device_fault() == 0
    _check_rows(Y, oracle.linear_g(X, qw, sc, z), kinds, f"group {group}")


@pytest.mark.parametrize("M", [1, 2, 10])
def test_awq_activation_scaling(cuda_lib, M):
    """w4a16_linear_awq: X' = bf16(x * r) formed ahead of (M <= 2) or inside (M >= 3) the X preparation."""
    N, K = 200, 1024
    kinds = [AWQ_KINDS[(m + 1) % len(AWQ_KINDS)] for m in range(M)]
    W = synth.weights_f32(15, synth.TAG_W, N, K)
    rng = np.random.default_rng(15)
    s = np.exp2(rng.uniform(-1.5, 1.5, size=K)).astype(np.float32)
    r = (1.0 / s.astype(np.float64)).astype(np.float32)
    pw = w4.PackedWeight(N, K)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    w4.quantize_pack_awq(torch.from_numpy(W).cuda(), torch.from_numpy(s).cuda(), pw.qweight, pw.scales,
                         pw.zeros, status)
    st, qw, sc, z = oracle.quantize_pack(oracle.awq_scale_weights(W, s))
    X = edge.activations_bf16(500 + M, kinds, K)
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(max(w4.workspace_bytes(M, N, K), 256), dtype=torch.uint8, device="cuda")
    w4.linear_awq(bits_to_dev_bf16(X), torch.from_numpy(r).cuda(), pw.qweight, pw.scales, pw.zeros, Y, ws,
                  path=w4.PATH_DECODE)
    torch.cuda.synchronize()
    assert int(status.item()) == 0 and st == oracle.OK and w4.device_fault() == 0
    Xs = oracle.awq_scale_activations(X, r)
    _check_rows(Y, oracle.linear(Xs, qw, sc, z), kinds, f"AWQ M={M}")


def test_prefill_gemm(cuda_lib):
    """M >= 64: BF16 tiles of (q - z) against BF16 X on the tensor cores (exact products, FP32 sums)."""
    N, K = 300, 1024
    kinds = [PREFILL_KINDS[m % len(PREFILL_KINDS)] for m in range(70)]
    pw, (qw, sc, z) = _pack(N, K, 16)
    X = edge.activations_bf16(600, kinds, K)
    Y = _linear(X, pw, w4.PATH_PREFILL)
    _check_rows(Y, oracle.linear(X, qw, sc, z), kinds, "prefill M=70")


@pytest.mark.parametrize("M", [1, 2, 3])
def test_w8a16(cuda_lib, M):
    """W8A16: the one-byte-code GEMV with the same digit representation of X."""
    N, K = 200, 1024
    W = synth.weights_f32(17, synth.TAG_W, N, K)
    pw = w4.PackedW8.from_float(torch.from_numpy(W).cuda())
    st, q, sc = oracle.w8_quantize(W)
    torch.cuda.synchronize()
    for start in range(0, len(ALL), M):
        kinds = [ALL[(start + i) % len(ALL)] for i in range(M)]
        X = edge.activations_bf16(700 + start, kinds, K)
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        ws = torch.zeros(max(w4.w8_workspace_bytes(M, N, K), 256), dtype=torch.uint8, device="cuda")
        w4.w8_linear(bits_to_dev_bf16(X), pw.qweight, pw.scales, Y, ws)
        torch.cuda.synchronize()
        assert w4.device_fault() == 0
        _check_rows(Y, oracle.w8_linear(X, q, sc), kinds, f"W8 M={M}")
