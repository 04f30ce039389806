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
