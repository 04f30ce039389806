"""Pins for the oracle's symmetric INT4 quantiser ("Quantization I: int8, int4,
the basics", Concept: a real value becomes an integer code through a scale
alone; the affine variants add a zero point).  The page's formula was lost in
extraction; the reading pinned here is signed codes q = clamp(rint(w/s), -8, 7)
with s = bf16(max|w| / 7) per group of 128, stored as the nibble q + 8 with the
zero point 8.  Every expected value below comes from a closed form, a brute
force over the 16 levels, or a library routine -- never from the oracle.
"""
import numpy as np

import oracle

S7 = 2.0 ** -7
LEVELS = np.arange(-8, 8, dtype=np.float64)


def _sym(W):
    st, qw, sc, z, clipped = oracle.quantize_pack(np.asarray(W, dtype=np.float32), with_clipped=True,
                                                  symmetric=True)
    return st, qw, sc, z, clipped


def _signed_codes(qw, K):
    return oracle.unpack(qw, K).astype(np.int64) - 8


def test_handworked_group_on_the_grid():
    """w = (k mod 15 - 7) 2^-7: max|w| = 7 2^-7, so s = 2^-7 exactly and the signed
    code is k mod 15 - 7 (nibble k mod 15 + 1)."""
    k = np.arange(128)
    w = ((k % 15) - 7) * S7
    st, qw, sc, z, clipped = _sym(w[None, :])
    assert st == oracle.OK
    assert int(sc[0, 0]) == 0x3C00  # bf16 bits of 2^-7
    assert int(z[0, 0]) == 8
    np.testing.assert_array_equal(oracle.unpack(qw, 128)[0], (k % 15) + 1)
    assert not clipped.any()


def test_handworked_ties_round_to_even():
    """With s = 2^-7 fixed by a 7 s entry: 2.5 s -> 2, -3.5 s -> -4, -0.5 s -> 0, 6.5 s -> 6,
    -6.5 s -> -6 (rint ties to even)."""
    w = np.zeros(128)
    w[0] = 7 * S7
    w[1:6] = np.array([2.5, -3.5, -0.5, 6.5, -6.5]) * S7
    st, qw, sc, z, _ = _sym(w[None, :])
    assert st == oracle.OK and int(sc[0, 0]) == 0x3C00
    q = _signed_codes(qw, 128)[0]
    np.testing.assert_array_equal(q[:6], [7, 2, -4, 0, 6, -6])
    assert np.all(q[6:] == 0)


def test_negative_extreme_and_zero_group():
    w = np.full((2, 128), 0.01)
    w[0, 3] = -7 * S7  # the magnitude maximum is negative: it takes code -7, not -8
    w[1] = 0.0
    st, qw, sc, z, _ = _sym(w)
    assert st == oracle.OK
    assert int(sc[0, 0]) == 0x3C00
    assert _signed_codes(qw, 128)[0, 3] == -7
    assert int(sc[1, 0]) == 0x3F80  # an all-zero group falls back to s = 1
    np.testing.assert_array_equal(oracle.unpack(qw, 128)[1], np.full(128, 8))
    np.testing.assert_array_equal(z, np.full((2, 1), 8))


def _bf16_nearest_brute(x):
    """Nearest BF16 to positive float64 x, ties to an even last bit, by trying the
    neighbouring bit patterns of its float32 truncation."""
    base = int(np.array([x], dtype=np.float32).view(np.uint32)[0] >> 16)
    best = None
    for c in (base - 1, base, base + 1, base + 2):
        v = float(np.array([c << 16], dtype=np.uint32).view(np.float32)[0])
        key = (abs(v - x), c & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return best[1]


def test_scale_is_nearest_bf16_of_max_over_seven():
    rng = np.random.default_rng(21)
    W = (rng.standard_normal((400, 128)) * rng.uniform(1e-3, 4.0, size=(400, 1))).astype(np.float32)
    st, qw, sc, z, _ = _sym(W)
    assert st == oracle.OK
    m = np.abs(W.astype(np.float64)).max(axis=1)
    want = [_bf16_nearest_brute(x / 7.0) for x in m]
    np.testing.assert_array_equal(sc[:, 0], np.array(want, dtype=np.uint16))


def test_codes_are_nearest_levels_brute_force():
    """Each weight takes the level of {-8..7} s nearest to it (ties to the even level);
    nothing clips, so |w - q s| <= s / 2; the magnitude maximum maps to +-7."""
    rng = np.random.default_rng(22)
    W = (rng.standard_normal((300, 128)) * rng.uniform(1e-2, 3.0, size=(300, 1))).astype(np.float32)
    W[::7, 5] *= 40.0  # outliers set the scale of some groups
    st, qw, sc, z, clipped = _sym(W)
    assert st == oracle.OK and not clipped.any()
    s = oracle.bf16_to_f64(sc[:, 0])[:, None]
    q = _signed_codes(qw, 128)
    w = W.astype(np.float64)
    dist = np.abs(w[:, :, None] - LEVELS[None, None, :] * s[:, :, None])
    best = dist.min(axis=2)
    np.testing.assert_array_equal(np.abs(w - q * s), best)
    ties = (dist == best[:, :, None]).sum(axis=2) > 1
    assert np.all(q[ties] % 2 == 0)
    assert np.all(np.abs(w - q * s) <= s / 2)
    am = np.argmax(np.abs(w), axis=1)
    np.testing.assert_array_equal(np.abs(q[np.arange(300), am]), 7)


def test_sign_symmetry():
    """Negating W negates every signed code and keeps every scale (no zero point)."""
    rng = np.random.default_rng(23)
    W = rng.standard_normal((64, 256)).astype(np.float32)
    _, qa, sa, _, _ = _sym(W)
    _, qb, sb, _, _ = _sym(-W)
    np.testing.assert_array_equal(sa, sb)
    np.testing.assert_array_equal(_signed_codes(qa, 256), -_signed_codes(qb, 256))


def test_requantize_grid_aligned_groups():
    """w = q s with BF16 s and signed codes reaching +-7 quantise back to exactly (s, q)."""
    rng = np.random.default_rng(24)
    G = 1500
    q = rng.integers(-7, 8, size=(G, 128))
    q[:, 0] = np.where(rng.integers(0, 2, size=G) == 1, 7, -7)
    sbits = rng.integers(0x3A00, 0x3E00, size=G).astype(np.uint16)
    s = oracle.bf16_to_f64(sbits)[:, None]
    W = (q * s).astype(np.float32)
    assert np.all(W.astype(np.float64) == q * s)
    st, qw, sc, z, _ = _sym(W)
    assert st == oracle.OK
    np.testing.assert_array_equal(sc[:, 0], sbits)
    np.testing.assert_array_equal(_signed_codes(qw, 128), q)


def test_linear_on_symmetric_weights_matches_library_matmul():
    """The oracle product on symmetric-packed weights equals X (q s)^T by numpy's FP64
    matmul, q and s built by hand."""
    rng = np.random.default_rng(25)
    N, K, M = 24, 384, 5
    q = rng.integers(-7, 8, size=(N, K))
    q[:, ::128] = 7
    sbits = rng.integers(0x3B00, 0x3D00, size=(N, K // 128)).astype(np.uint16)
    s = np.repeat(oracle.bf16_to_f64(sbits), 128, axis=1)
    W = (q * s).astype(np.float32)
    st, qw, sc, z, _ = _sym(W)
    assert st == oracle.OK
    xbits = (np.array(rng.standard_normal((M, K)), dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)
    want = oracle.bf16_to_f64(xbits) @ (q * s).T
    got = oracle.linear(xbits, qw, sc, z)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_nonfinite_status():
    W = np.zeros((2, 256), dtype=np.float32)
    W[1, 200] = np.inf
    st, *_ = _sym(W)
    assert st == oracle.ERR_NONFINITE
