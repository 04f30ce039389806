"""Pins for the oracle's AWQ equivalence transform ("Axe Corsa 28B" model card,
"How the Compression Works", Stage 1; "Weight-Only Quantization and Mixed
Precision", section 3): input channel k of W is multiplied by s_k and the same
channel of X by s_k^-1, so X W^T is unchanged in exact arithmetic, and rounding
the rescaled weights loses less on the salient (large-activation) channels.

Expected values come from exact power-of-two identities, brute-force nearest
representable values, numpy's FP64 matmul, and the pages' claim of lower output
error -- never from the oracle itself.
"""
import numpy as np

import oracle
import synth


def _bf16_bits_of(x: np.ndarray) -> np.ndarray:
    """Truncation of float32 values that are already BF16-representable."""
    return (np.asarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_power_of_two_scales_are_an_exact_equivalence():
    """With s_k = 2^e_k and r_k = 2^-e_k every rescaled element is exact, so the
    library FP64 product of the transformed operands equals the original bit for bit;
    a transform applied along the wrong axis would break the identity."""
    rng = np.random.default_rng(31)
    N, K, M = 48, 384, 7
    e = rng.integers(-3, 4, size=K)
    s = np.ldexp(1.0, e).astype(np.float32)
    r = np.ldexp(1.0, -e).astype(np.float32)
    W = synth.weights_f32(3, synth.TAG_W, N, K)
    X = synth.activations_bf16(4, M, K)
    Wp = oracle.awq_scale_weights(W, s)
    Xp = oracle.awq_scale_activations(X, r)
    np.testing.assert_array_equal(Wp.astype(np.float64), W.astype(np.float64) * np.ldexp(1.0, e)[None, :])
    np.testing.assert_array_equal(oracle.bf16_to_f64(Xp), oracle.bf16_to_f64(X) * np.ldexp(1.0, -e)[None, :])
    lhs = oracle.bf16_to_f64(Xp) @ Wp.astype(np.float64).T
    rhs = oracle.bf16_to_f64(X) @ W.astype(np.float64).T
    np.testing.assert_array_equal(lhs, rhs)


def test_weight_transform_rounds_to_the_nearest_float():
    """W' is the binary32 value nearest to w s (neither float neighbour is closer)."""
    rng = np.random.default_rng(32)
    W = synth.weights_f32(5, synth.TAG_W, 64, 256)
    s = rng.uniform(0.2, 5.0, size=256).astype(np.float32)
    Wp = oracle.awq_scale_weights(W, s)
    exact = W.astype(np.float64) * s.astype(np.float64)[None, :]
    err = np.abs(Wp.astype(np.float64) - exact)
    for nb in (np.nextafter(Wp, np.float32(np.inf)), np.nextafter(Wp, np.float32(-np.inf))):
        assert np.all(err <= np.abs(nb.astype(np.float64) - exact))
    assert np.all(err <= np.abs(exact) * 2.0 ** -24)


def test_activation_transform_rounds_to_the_nearest_bf16():
    """X' is the BF16 value nearest to x r, checked against the two BF16 neighbours."""
    rng = np.random.default_rng(33)
    M, K = 16, 512
    X = synth.activations_bf16(6, M, K)
    r = (1.0 / rng.uniform(0.2, 5.0, size=K)).astype(np.float32)
    Xp = oracle.awq_scale_activations(X, r)
    exact = oracle.bf16_to_f64(X) * r.astype(np.float64)[None, :]
    got = oracle.bf16_to_f64(Xp)
    err = np.abs(got - exact)
    mag = Xp & 0x7FFF
    for step in (1, -1):
        nb_bits = (Xp & 0x8000) | np.clip(mag.astype(np.int64) + step, 0, 0x7F7F).astype(np.uint16)
        assert np.all(err <= np.abs(oracle.bf16_to_f64(nb_bits) - exact))
    assert np.all(err <= np.abs(exact) * 2.0 ** -8)


def test_rescaling_salient_channels_lowers_the_output_error():
    """The pages' claim: scaling the weights of the large-activation channels up
    (s_k = mean|x_k|^0.5, normalised) before 4-bit rounding, and the activations
    down, gives a smaller output error than rounding W directly."""
    N, K, M = 256, 1024, 64
    W = synth.weights_f32(7, synth.TAG_W, N, K)
    X = synth.activations_bf16(8, M, K)
    xf = oracle.bf16_to_f64(X)
    imp = np.abs(xf).mean(axis=0)
    s64 = np.sqrt(imp)
    s64 /= np.exp(np.log(s64).mean())
    s = s64.astype(np.float32)
    r = (1.0 / s.astype(np.float64)).astype(np.float32)
    y_exact = xf @ W.astype(np.float64).T

    st, qw, sc, z = oracle.quantize_pack(W)
    y_rtn = oracle.linear(X, qw, sc, z)
    Wp = oracle.awq_scale_weights(W, s)
    Xp = oracle.awq_scale_activations(X, r)
    st2, qw2, sc2, z2 = oracle.quantize_pack(Wp)
    y_awq = oracle.linear(Xp, qw2, sc2, z2)
    assert st == st2 == oracle.OK
    e_rtn = np.linalg.norm(y_rtn - y_exact)
    e_awq = np.linalg.norm(y_awq - y_exact)
    assert e_awq < 0.8 * e_rtn, (e_awq, e_rtn)
    # the transform itself (no quantisation) is an equivalence up to its roundings
    y_equiv = oracle.bf16_to_f64(Xp) @ Wp.astype(np.float64).T
    assert np.linalg.norm(y_equiv - y_exact) < 0.05 * e_awq
