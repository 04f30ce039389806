"""The seeded input generator: deterministic, counter-addressable, and drawing
the stated distributions (W ~ N(0, 0.02); X ~ N(0, 1) with 1% of input
channels scaled x20)."""
import math

import numpy as np
import torch

import synth


def test_ln_and_cos_match_libm():
    rng = np.random.default_rng(0)
    for u in list(rng.random(2000)) + [1.0, 0.5, 2.0 ** -53, 0.7071067811865476, 1 - 2.0 ** -53]:
        if u <= 0:
            continue
        assert abs(synth.ln(u) - math.log(u)) <= 4e-16 * max(1.0, abs(math.log(u)))
    for u in list(rng.random(2000)) + [0.0, 0.125, 0.25, 0.5, 0.75, 0.999]:
        assert abs(synth.cos2pi(u) - math.cos(2 * math.pi * u)) <= 1e-15


def test_weights_deterministic_and_addressable():
    a = synth.weights_f32(3, synth.TAG_W, 64, 256)
    b = synth.weights_f32(3, synth.TAG_W, 64, 256)
    np.testing.assert_array_equal(a, b)
    rows = synth.weight_rows_f32(3, synth.TAG_W, 256, [63, 0, 17])
    np.testing.assert_array_equal(rows, a[[63, 0, 17]])
    c = synth.weights_f32(4, synth.TAG_W, 64, 256)
    assert not np.array_equal(a, c)
    d = synth.weights_f32(3, synth.TAG_X, 64, 256)
    assert not np.array_equal(a, d)


def test_weight_moments():
    W = synth.weights_f32(1, synth.TAG_W, 1024, 1024).astype(np.float64)
    assert abs(W.mean()) < 1e-4
    assert abs(W.std() - 0.02) < 1e-4
    kurt = ((W / W.std()) ** 4).mean()
    assert abs(kurt - 3.0) < 0.05
    # tails: P(|z| > 3) = 0.0027
    assert abs((np.abs(W) > 0.06).mean() - 0.0027) < 0.0005


def test_activations_outliers():
    for K in (4096, 5120, 8192, 25600, 28672):
        assert synth.n_outliers(K) == round(K / 100 + 1e-9)
    K = 8192
    ch = synth.outlier_channels(5, K)
    assert ch.size == 82 and np.unique(ch).size == 82 and ch.min() >= 0 and ch.max() < K
    X = synth.activations_bf16(5, 64, K)
    x = torch.from_numpy(X.view(np.int16)).view(torch.bfloat16).double().numpy()
    mask = np.zeros(K, bool)
    mask[ch] = True
    assert abs(x[:, mask].std() / x[:, ~mask].std() - 20.0) < 1.0
    assert abs(x[:, ~mask].std() - 1.0) < 0.01


def test_bf16_formatting_matches_library_on_floats():
    rng = np.random.default_rng(1)
    f = (rng.standard_normal(5000) * 10.0 ** rng.integers(-20, 20, 5000)).astype(np.float32)
    lib_bits = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ours = np.array([synth.bf16_bits(float(v)) for v in f], dtype=np.uint16)
    np.testing.assert_array_equal(ours, lib_bits)
