"""The integer representation of X that the decode kernels multiply, checked on the
host in numpy: per group of 128 activations,
E = the exponent of the largest |x|, x_int = rint(x 2^(21 - E)) written in
balanced base 256 (x_int = 65536 d2 + 256 d1 + d0, every digit in [-128, 127]).
The claims the kernels rely on: the digits fit signed bytes and recompose x_int
exactly; values within 2^14 of the group maximum are represented exactly; every
value is within half a step, 2^(E - 22), of its representation; and the products
with 4-bit codes summed over a group stay exact in int32 per digit plane.
"""
import numpy as np

import synth


def _bf16_to_f32(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _digits(xb):
    """xb: BF16 bits of one group (128 values) -> (E, x_int, d0, d1, d2)."""
    amax = int((xb & 0x7FFF).max())
    ef = amax >> 7
    E = -127 if ef == 0 else ef - 127
    x = _bf16_to_f32(xb).astype(np.float64)
    xi = np.rint(np.ldexp(x, 21 - E)).astype(np.int64)
    d0 = ((xi + 128) & 255) - 128
    t = (xi - d0) >> 8
    d1 = ((t + 128) & 255) - 128
    d2 = (t - d1) >> 8
    return E, x, xi, d0, d1, d2


def test_digits_recompose_and_fit_signed_bytes():
    X = synth.activations_bf16(3, 64, 4096).reshape(-1, 128)
    for xb in X[:2000]:
        E, x, xi, d0, d1, d2 = _digits(xb)
        for d in (d0, d1, d2):
            assert d.min() >= -128 and d.max() <= 127
        np.testing.assert_array_equal(65536 * d2 + 256 * d1 + d0, xi)
        assert np.abs(xi).max() < 2 ** 22


def test_exact_within_2_14_of_the_maximum_and_half_step_elsewhere():
    rng = np.random.default_rng(5)
    for _ in range(500):
        scale = 2.0 ** rng.integers(-30, 30)
        x = rng.standard_normal(128) * scale * np.exp(rng.uniform(-12, 0, size=128))
        xb = (x.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
        E, xv, xi, *_ = _digits(xb)
        rep = np.ldexp(xi.astype(np.float64), E - 21)
        big = np.abs(xv) >= 2.0 ** (E - 14)
        np.testing.assert_array_equal(rep[big], xv[big])
        assert np.all(np.abs(rep - xv) <= 2.0 ** (E - 22))


def test_plane_sums_stay_exact_in_int32():
    """sum over a group of q d_p with q in [0, 15] (INT4) or [-127, 127] (INT8): at most
    128 * 15 * 128 or 128 * 127 * 128 in magnitude, and 256 P1 + P0 below 2^31."""
    worst4 = 128 * 15 * 128
    worst8 = 128 * 127 * 128
    assert worst4 < 2 ** 21 and worst8 < 2 ** 21
    assert 256 * worst8 + worst8 < 2 ** 31


# ---------------------------------------------------------------------------------------------
# The one-token GEMV's variant.  Its A operand takes the two halves of a packed word as bytes without a
# shift: w & 0x0F0F0F0F holds codes 0, 2, 4, 6 of the word and w & 0xF0F0F0F0 holds 16 times codes 1, 3, 5, 7.
# The activations of the odd codes (K odd) are therefore expressed with four fewer fractional bits,
# x_int = rint(x 2^(17 - E)), those of the even codes as above, rint(x 2^(21 - E)), and the group's
# represented dot product is 2^(E - 21) (sum_even q x_int + sum_odd 16 q x_int).  Claims checked here: the
# odd values are exact within 2^10 of the group maximum and within half a step, 2^(E - 18), elsewhere; the
# digits fit signed bytes and recompose; the plane sums (bytes of at most 240 against digits of at most
# 128) stay below 2^22, the range in which the accumulators' bias 1.5 2^23 converts them exactly; and the
# represented product differs from the exact one by no more than the half steps allow.


def _one_token_ints(xb):
    """xb: BF16 bits of one group -> (E, x, x_int) with the even/odd scalings of the one-token kernel."""
    amax = int((xb & 0x7FFF).max())
    ef = amax >> 7
    E = -127 if ef == 0 else ef - 127
    x = _bf16_to_f32(xb).astype(np.float64)
    k = np.arange(x.size)
    shift = np.where(k % 2 == 1, 17 - E, 21 - E)
    xi = np.rint(np.ldexp(x, shift)).astype(np.int64)
    return E, x, xi, k % 2 == 1


def _balanced_digits(xi):
    d0 = ((xi + 128) & 255) - 128
    t = (xi - d0) >> 8
    d1 = ((t + 128) & 255) - 128
    d2 = (t - d1) >> 8
    return d0, d1, d2


def test_one_token_odd_codes_exact_within_2_10_and_half_step_elsewhere():
    rng = np.random.default_rng(11)
    for _ in range(500):
        scale = 2.0 ** rng.integers(-30, 30)
        x = rng.standard_normal(128) * scale * np.exp(rng.uniform(-12, 0, size=128))
        xb = (x.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
        E, xv, xi, odd = _one_token_ints(xb)
        rep = np.where(odd, np.ldexp(xi.astype(np.float64), E - 17), np.ldexp(xi.astype(np.float64), E - 21))
        exact_odd = odd & (np.abs(xv) >= 2.0 ** (E - 10))
        exact_even = ~odd & (np.abs(xv) >= 2.0 ** (E - 14))
        np.testing.assert_array_equal(rep[exact_odd], xv[exact_odd])
        np.testing.assert_array_equal(rep[exact_even], xv[exact_even])
        assert np.all(np.abs(rep - xv)[odd] <= 2.0 ** (E - 18))
        assert np.all(np.abs(rep - xv)[~odd] <= 2.0 ** (E - 22))


def test_one_token_digits_and_plane_sums_on_edge_activations():
    from synth import edge
    kinds = list(edge.KINDS)
    X = edge.activations_bf16(21, kinds, 1024)
    rng = np.random.default_rng(12)
    worst = 64 * 15 * 128 + 64 * 240 * 128  # even bytes q, odd bytes 16 q, digits of magnitude <= 128
    assert worst < 2 ** 22
    bias = np.float32(12582912.0)  # 1.5 2^23
    for row in X:
        for xb in row.reshape(-1, 128):
            E, x, xi, odd = _one_token_ints(xb)
            assert np.abs(xi[odd]).max(initial=0) < 2 ** 18 and np.abs(xi[~odd]).max(initial=0) < 2 ** 22
            d0, d1, d2 = _balanced_digits(xi)
            for d in (d0, d1, d2):
                assert d.min() >= -128 and d.max() <= 127
            np.testing.assert_array_equal(65536 * d2 + 256 * d1 + d0, xi)
            q = rng.integers(0, 16, size=128)
            a = np.where(odd, 16 * q, q)  # the A bytes
            planes = [int((a * d).sum()) for d in (d0, d1, d2)]
            for P in planes:
                assert abs(P) <= worst
                # the accumulator starts at the bits of 1.5 2^23 and ends as the FP32 number 1.5 2^23 + P
                assert float(np.float32(bias + np.float32(P)) - bias) == P
            # the integer identity the fold relies on, and the product within the half-step bound
            assert 65536 * planes[2] + 256 * planes[1] + planes[0] == int((a * xi).sum())
            represented = np.ldexp(float((a * xi).sum()), E - 21)
            exact = float((q * x).sum())
            bound = float((q[odd] * 2.0 ** (E - 18)).sum() + (q[~odd] * 2.0 ** (E - 22)).sum())
            assert abs(represented - exact) <= bound + 1e-300


# ---------------------------------------------------------------------------------------------
# The same scheme as the GPU writes it: the 2-16-token integer GEMV prepares each launch's digit
# rows once, in its caller's workspace, and reads them back with bulk copies.  White-box check of
# that preparation, bit for bit, against the host statement above: the workspace layout is
# [256 KB of split-K counters][per group g: digit rows of 128 bytes, then (sum x_int, 2^(E - 21)) per
# token as FP32].  Within a row, bytes 8w .. 8w + 3 hold the digits of codes 0, 2, 4, 6 of packed
# word w (K = 128 g + 8 w + {0, 2, 4, 6}) and bytes 8w + 4 .. 8w + 7 those of codes 1, 3, 5, 7.
# Row of plane p, token m: 2m + p (p < 2) or 8 + 2m (p = 2) for 4-token tiles, p NT + m otherwise.

import pytest  # noqa: E402


def _mt_row(nt, p, m):
    return (2 * m + p if p < 2 else 8 + 2 * m) if nt == 4 else p * nt + m


@pytest.mark.gpu
@pytest.mark.parametrize("M,nt", [(2, 4), (3, 4), (4, 4), (6, 8), (8, 8), (12, 16), (16, 16)])
def test_gpu_digit_rows_match_the_scheme(cuda_lib, M, nt):
    import torch
    import weight_only_int4_linear_b200 as w4
    from tests._parity import bits_to_dev_bf16
    from synth import edge
    N, K = 256, 1024
    G = K // 128
    kinds = [edge.KINDS[m % len(edge.KINDS)] for m in range(M)]
    kinds[0] = "control"
    Xb = edge.activations_bf16(77 + M, kinds, K)
    W = synth.weights_f32(5, synth.TAG_W, N, K)
    pw = w4.PackedWeight.from_float(torch.from_numpy(W).cuda())
    nbytes = w4.workspace_bytes(M, N, K)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    w4.linear(bits_to_dev_bf16(Xb), pw.qweight, pw.scales, pw.zeros, Y, ws, path=w4.PATH_DECODE)
    torch.cuda.synchronize()
    rows = {4: 16, 8: 24, 16: 48}[nt]
    xbytes = rows * 128 + 8 * nt
    counters = 256 * 1024
    raw = ws.cpu().numpy()
    assert not raw[:counters].any()  # every counter back at zero
    order = np.array([[8 * w + i for i in (0, 2, 4, 6, 1, 3, 5, 7)] for w in range(16)]).reshape(-1)
    for g in range(G):
        blk = raw[counters + g * xbytes: counters + (g + 1) * xbytes]
        planes = blk[: rows * 128].reshape(rows, 128).view(np.int8)
        ext = blk[rows * 128:].view(np.float32)
        used = np.zeros(rows, dtype=bool)
        for m in range(nt):
            if m < M:
                E, x, xi, d0, d1, d2 = _digits(Xb[m, 128 * g:128 * (g + 1)])
                want = [d0, d1, d2]
                assert ext[2 * m] == float(xi.sum()), (g, m)
                assert ext[2 * m + 1] == np.ldexp(1.0, E - 21), (g, m)
            else:
                want = [np.zeros(128, dtype=np.int64)] * 3
                assert ext[2 * m] == 0 and ext[2 * m + 1] == 0
            for p in range(3):
                r = _mt_row(nt, p, m)
                used[r] = True
                np.testing.assert_array_equal(planes[r].astype(np.int64), want[p][order], err_msg=f"g={g} m={m} p={p}")
        assert not planes[~used].any()  # padding rows stay zero
