"""Pins for the oracle's W8A16 arithmetic ("Weight-Only Quantization and Mixed
Precision", sections 5 and 8: INT8 weights, 16-bit activations, no grouping;
"Weight-Only Quantisation", Notes).  The pages give no INT8 formula; the reading
pinned is symmetric per output channel: s_n = bf16(max_k |w[n][k]| / 127),
q = clamp(rint(w / s_n), -127, 127), w_hat = q s_n.  Expected values come from
closed forms, brute force over the 255 levels, numpy's FP64 matmul and the
pages' compression ratio -- never from the oracle.
"""
import numpy as np

import oracle

S7 = 2.0 ** -7
LEVELS = np.arange(-127, 128, dtype=np.float64)


def _bf16_nearest_brute(x):
    base = int(np.array([x], dtype=np.float32).view(np.uint32)[0] >> 16)
    best = None
    for c in (base - 1, base, base + 1, base + 2):
        v = float(np.array([c << 16], dtype=np.uint32).view(np.float32)[0])
        key = (abs(v - x), c & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return best[1]


def test_handworked_row_on_the_grid():
    k = np.arange(256)
    w = ((k % 255) - 127) * S7
    st, q, sc = oracle.w8_quantize(w[None, :])
    assert st == oracle.OK
    assert int(sc[0]) == 0x3C00  # 2^-7: max|w| = 127 2^-7
    np.testing.assert_array_equal(q[0], (k % 255) - 127)


def test_handworked_ties_round_to_even():
    w = np.zeros(128)
    w[0] = 127 * S7
    w[1:6] = np.array([2.5, -3.5, 126.5, -0.5, -126.5]) * S7
    st, q, sc = oracle.w8_quantize(w[None, :])
    assert st == oracle.OK and int(sc[0]) == 0x3C00
    np.testing.assert_array_equal(q[0, :6], [127, 2, -4, 126, 0, -126])


def test_negative_extreme_zero_row_and_status():
    W = np.full((3, 128), 0.01, dtype=np.float32)
    W[0, 7] = -127 * S7
    W[1] = 0.0
    st, q, sc = oracle.w8_quantize(W[:2])
    assert st == oracle.OK
    assert int(sc[0]) == 0x3C00 and q[0, 7] == -127
    assert int(sc[1]) == 0x3F80 and not q[1].any()
    W[2, 3] = np.nan
    st, *_ = oracle.w8_quantize(W)
    assert st == oracle.ERR_NONFINITE


def test_scale_is_nearest_bf16_of_max_over_127():
    rng = np.random.default_rng(61)
    W = (rng.standard_normal((300, 384)) * rng.uniform(1e-3, 5.0, size=(300, 1))).astype(np.float32)
    st, q, sc = oracle.w8_quantize(W)
    m = np.abs(W.astype(np.float64)).max(axis=1)
    np.testing.assert_array_equal(sc, np.array([_bf16_nearest_brute(x / 127.0) for x in m], dtype=np.uint16))


def test_codes_are_nearest_levels_brute_force():
    rng = np.random.default_rng(62)
    W = (rng.standard_normal((40, 512)) * 0.02).astype(np.float32)
    W[::5, 17] *= 30.0
    st, q, sc, clipped = oracle.w8_quantize(W, with_clipped=True)
    assert st == oracle.OK and not clipped.any()
    s = oracle.bf16_to_f64(sc)[:, None]
    w = W.astype(np.float64)
    qq = q.astype(np.float64)
    dist = np.abs(w[:, :, None] - LEVELS[None, None, :] * s[:, :, None])
    best = dist.min(axis=2)
    np.testing.assert_array_equal(np.abs(w - qq * s), best)
    ties = (dist == best[:, :, None]).sum(axis=2) > 1
    assert np.all(q[ties] % 2 == 0)
    am = np.argmax(np.abs(w), axis=1)
    np.testing.assert_array_equal(np.abs(q[np.arange(40), am]), 127)


def test_requantize_grid_aligned_rows():
    rng = np.random.default_rng(63)
    N, K = 500, 256
    qw = rng.integers(-127, 128, size=(N, K))
    qw[:, 3] = np.where(rng.integers(0, 2, size=N) == 1, 127, -127)
    sbits = rng.integers(0x3A00, 0x3E00, size=N).astype(np.uint16)
    s = oracle.bf16_to_f64(sbits)[:, None]
    W = (qw * s).astype(np.float32)
    assert np.all(W.astype(np.float64) == qw * s)
    st, q, sc = oracle.w8_quantize(W)
    np.testing.assert_array_equal(sc, sbits)
    np.testing.assert_array_equal(q, qw)


def test_linear_matches_library_matmul():
    rng = np.random.default_rng(64)
    M, N, K = 6, 40, 640
    qw = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    sbits = rng.integers(0x3B00, 0x3D00, size=N).astype(np.uint16)
    xbits = (rng.standard_normal((M, K)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    want = oracle.bf16_to_f64(xbits) @ (qw.astype(np.float64) * oracle.bf16_to_f64(sbits)[:, None]).T
    got = oracle.w8_linear(xbits, qw, sbits)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_storage_is_half_of_bf16():
    """The selection matrix's 2x weight compression for INT8 (4x for INT4): one byte per
    weight plus one BF16 scale per row."""
    N, K = 8192, 8192
    w8 = N * K + 2 * N
    assert abs(N * K * 2 / w8 - 2.0) < 1e-3
