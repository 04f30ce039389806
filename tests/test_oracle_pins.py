"""Pins for the FP64 oracle: checked against hand-worked values, closed forms,
library routines and invariants of the scheme -- never against itself.

Sources: "Axe Corsa 28B" model card ("How the Compression Works", "What the
Tensor Types Tell You", "Storage Cost"); "Quantization I: int8, int4, the
basics" (Concept).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "handworked_groups.json")
S7 = 2.0 ** -7


def _case_weights(name: str) -> np.ndarray:
    k = np.arange(128)
    if name == "grid_aligned":
        w = ((k % 16) - 5) * S7
    elif name == "ties_to_even":
        w = ((k % 12) - 4) * S7
        w[0], w[1], w[2] = -4.5 * S7, 10.5 * S7, 2.5 * S7
    elif name == "negative_zero_point":
        w = ((k % 16) + 3) * S7
    elif name == "all_levels_from_zero":
        w = (k % 16) * S7
    elif name == "constant_group":
        w = np.full(128, 0.3)
    elif name == "zero_group":
        w = np.zeros(128)
    else:
        raise KeyError(name)
    return w.astype(np.float32)


def _case_codes(name: str) -> np.ndarray:
    k = np.arange(128)
    if name in ("grid_aligned", "negative_zero_point", "all_levels_from_zero"):
        return (k % 16).astype(np.uint8)
    if name == "ties_to_even":
        c = (k % 12).astype(np.uint8)
        c[0], c[1], c[2] = 0, 14, 6
        return c
    return np.zeros(128, dtype=np.uint8)


@pytest.fixture(scope="module")
def golden():
    with open(GOLDEN) as f:
        return json.load(f)


def test_handworked_groups(golden):
    for case in golden["cases"]:
        name = case["name"]
        W = _case_weights(name)[None, :]
        st, qw, sc, z = oracle.quantize_pack(W)
        assert st == oracle.OK, name
        assert int(sc[0, 0]) == int(case["scale_bits"], 16), name
        assert int(z[0, 0]) == case["zero"], name
        codes = oracle.unpack(qw, 128)[0]
        np.testing.assert_array_equal(codes, _case_codes(name), err_msg=name)
        if "words" in case:
            expect = [int(h, 16) for h in case["words"]] * 8
            assert [int(v) for v in qw[0]] == expect, name
        wh = oracle.dequant(qw, sc, z, 128)[0]
        if case["w_hat_equals_w"]:
            np.testing.assert_array_equal(wh, W[0].astype(np.float64), err_msg=name)
        if "w_hat_value" in case:
            assert np.all(wh == case["w_hat_value"]), name
        if "max_abs_error_over_s" in case:
            s = oracle.bf16_value(int(sc[0, 0]))
            assert np.max(np.abs(wh - W[0])) / s == case["max_abs_error_over_s"], name
        if "y_ones" in case:
            X = np.full((1, 128), 0x3F80, dtype=np.uint16)  # BF16 1.0
            Y = oracle.linear(X, qw, sc, z)
            assert Y[0, 0] == case["y_ones"], name
        if "y_ones_bf16_bits" in case:
            assert oracle.bf16_round(Y[0, 0]) == int(case["y_ones_bf16_bits"], 16)


def test_tiny_matmul(golden):
    t = golden["tiny_matmul"]
    W = np.stack([_case_weights(n) for n in t["rows"]])
    st, qw, sc, z = oracle.quantize_pack(W)
    assert st == oracle.OK
    X = np.zeros((2, 128), dtype=np.uint16)
    X[0, :] = 0x3F80
    X[1, 5] = 0x3F80
    Y = oracle.linear(X, qw, sc, z)
    np.testing.assert_array_equal(Y, np.array(t["Y"]))
    Ys = oracle.linear_sampled(X, qw, sc, z, [1, 0], [2, 0, 1])
    np.testing.assert_array_equal(Ys, np.array(t["Y"])[[1, 0]][:, [2, 0, 1]])


def test_storage_cost(golden):
    """4.375 bits per weight from the packed buffers' sizes (model card, Storage Cost)."""
    N, K = 64, 1024
    W = synth.weights_f32(7, synth.TAG_W, N, K)
    st, qw, sc, z = oracle.quantize_pack(W)
    bits = 8 * (qw.nbytes + sc.nbytes + z.nbytes) / (N * K)
    assert bits == golden["storage_cost"]["bits_per_weight"]
    assert abs(16 / bits - golden["storage_cost"]["compression_vs_bf16"]) < 1e-12
    assert round(16 / bits, 2) == 3.66


def test_bf16_round_cases():
    cases = [
        (1.0 + 2.0 ** -8, 0x3F80),              # tie -> even (1.0)
        (1.0 + 3 * 2.0 ** -8, 0x3F82),          # tie -> even (1 + 2^-6)
        (1.0 + 2.0 ** -8 + 2.0 ** -30, 0x3F81),  # just above the tie
        (-2.5, 0xC020),
        (2.0 ** -133, 0x0001),                  # smallest BF16 subnormal
        (1.5 * 2.0 ** -133, 0x0002),            # subnormal tie -> even
        (0.5 * 2.0 ** -133, 0x0000),            # tie -> even (zero)
        (0.75 * 2.0 ** -133, 0x0001),
        (2.0 ** -126, 0x0080),                  # smallest normal
        (float.fromhex("0x1.FEp127"), 0x7F7F),  # largest finite
        (float.fromhex("0x1.FFp127"), 0x7F80),  # tie past the largest finite -> inf
        (0.0, 0x0000),
        (-0.0, 0x8000),
    ]
    for x, bits in cases:
        assert oracle.bf16_round(x) == bits, (x, hex(oracle.bf16_round(x)))


def test_bf16_round_matches_library_on_floats():
    """For binary32 inputs the BF16 rounding must equal torch's float->bf16 (RNE)."""
    rng = np.random.default_rng(3)
    f = np.concatenate([
        (rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000)).astype(np.float32),
        np.frombuffer(rng.integers(0, 2 ** 32, 20000, dtype=np.uint64).astype(np.uint32).tobytes(),
                      dtype=np.float32),
    ])
    assert f.dtype == np.float32
    f = f[np.isfinite(f)]
    lib_bits = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ours = np.array([oracle.bf16_round(float(v)) for v in f], dtype=np.uint16)
    np.testing.assert_array_equal(ours, lib_bits)


def _random_groups(n_groups: int, seed: int) -> np.ndarray:
    """Seeded N(0, 0.02) groups plus shifted and rescaled ones (non-zero means,
    one-signed groups with negative zero points, wide and tiny ranges)."""
    W = synth.weights_f32(seed, synth.TAG_W, n_groups, 128)
    rng = np.random.default_rng(seed)
    shift = rng.choice([0.0, 0.05, -0.05, 2.5, -10.0, 10.0], size=(n_groups, 1)).astype(np.float32)
    scale = rng.choice([1.0, 1e-3, 40.0, 1e-20], size=(n_groups, 1)).astype(np.float32)
    return ((W + shift * np.float32(0.02)) * scale).astype(np.float32)


def test_invariants_random_groups():
    W = _random_groups(10000, 11)
    st, qw, sc, z, clipped = oracle.quantize_pack(W, with_clipped=True)
    assert st == oracle.OK
    codes = oracle.unpack(qw, 128)
    assert codes.max() <= 15
    s = oracle.bf16_to_f64(sc[:, 0])[:, None]
    wh = oracle.dequant(qw, sc, z, 128)
    err = np.abs(wh - W.astype(np.float64))
    ok = clipped == 0
    # per-group reconstruction error <= s/2 for unclipped values (exact comparison)
    assert np.all(err[ok] <= (s / 2 * np.ones_like(err))[ok])
    # clipping is rare (only from BF16 rounding of s at the top of the range)
    assert clipped.mean() < 1e-3
    # the group minimum maps to code 0 (rint is odd-symmetric, z unclamped)
    argmin = np.argmin(W, axis=1)
    assert np.all(codes[np.arange(W.shape[0]), argmin] == 0)
    # some groups have zero points outside [0, 15] (one-signed groups)
    assert (z < 0).any() and (z > 15).any()


def test_pack_unpack_roundtrip():
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 16, size=(37, 512), dtype=np.uint8)
    qw = oracle.pack_codes(codes)
    np.testing.assert_array_equal(oracle.unpack(qw, 512), codes)
    # nibble order: low nibble first along K
    assert int(qw[0, 0]) == sum(int(codes[0, i]) << (4 * i) for i in range(8))


def test_requantize_grid_aligned_groups():
    """Weights built on the grid, (q - z) s with BF16 s and codes spanning 0..15,
    quantise back to exactly the same (s, z, q)."""
    rng = np.random.default_rng(9)
    G = 2000
    codes = rng.integers(0, 16, size=(G, 128), dtype=np.uint8)
    codes[:, 0] = 0
    codes[:, 1] = 15
    zs = rng.integers(-20, 36, size=G)
    sbits = (rng.integers(0x3A00, 0x3E00, size=G)).astype(np.uint16)  # BF16 scales ~ 5e-4 .. 0.125
    s = oracle.bf16_to_f64(sbits)
    W = ((codes.astype(np.float64) - zs[:, None]) * s[:, None]).astype(np.float32)
    assert np.all(W.astype(np.float64) == (codes.astype(np.float64) - zs[:, None]) * s[:, None])
    st, qw, sc, z = oracle.quantize_pack(W)
    assert st == oracle.OK
    np.testing.assert_array_equal(sc[:, 0], sbits)
    np.testing.assert_array_equal(z[:, 0], zs)
    np.testing.assert_array_equal(oracle.unpack(qw, 128), codes)


def test_status_codes():
    W = np.zeros((2, 256), dtype=np.float32)
    W[1, 7] = np.nan
    st, *_ = oracle.quantize_pack(W)
    assert st == oracle.ERR_NONFINITE
    W = np.zeros((1, 256), dtype=np.float32)
    W[0, :128] = np.float32(1e30)
    W[0, 0] = np.float32(1e30 * (1 - 2 ** -20))
    st, *_ = oracle.quantize_pack(W)
    # s ~ 1e30 * 2^-20 / 15 and -lo/s ~ 1.6e7: fits int32
    assert st == oracle.OK
    W[0, 0] = np.float32(1e30 * (1 - 2 ** -23))
    W[0, 1] = np.float32(-1e30)
    st, *_ = oracle.quantize_pack(W)
    assert st == oracle.OK
    # A zero point outside int32 cannot arise from finite binary32 groups: hi - lo
    # is at least one ulp of the larger magnitude, so |lo| / s stays below
    # about 15 * 2^24.  Both sides still check it.
    W = np.zeros((1, 128), dtype=np.float32)
    W[0, :] = np.float32(3e38)
    W[0, 0] = np.nextafter(np.float32(3e38), np.float32(0))
    st, qw, sc, z = oracle.quantize_pack(W)
    assert st == oracle.OK and abs(int(z[0, 0])) < 15 * 2 ** 24
    W = np.zeros((1, 100), dtype=np.float32)
    st, *_ = oracle.quantize_pack(W)
    assert st == oracle.ERR_SHAPE


def test_linear_matches_library_matmul():
    """With W_hat materialised, the layer is a dense matmul: compare with numpy's
    FP64 matmul (a library routine) on small shapes."""
    for (M, N, K, seed) in [(1, 5, 128, 1), (3, 17, 256, 2), (8, 64, 1024, 3)]:
        W = synth.weights_f32(seed, synth.TAG_W, N, K)
        X = synth.activations_bf16(seed, M, K)
        st, qw, sc, z = oracle.quantize_pack(W)
        Y = oracle.linear(X, qw, sc, z)
        ref = oracle.bf16_to_f64(X) @ oracle.dequant(qw, sc, z, K).T
        np.testing.assert_allclose(Y, ref, rtol=1e-13, atol=1e-13 * np.abs(ref).max())
        m_idx, n_idx = [M - 1, 0], [N - 1, 0, N // 2]
        np.testing.assert_array_equal(oracle.linear_sampled(X, qw, sc, z, m_idx, n_idx),
                                      Y[np.ix_(m_idx, n_idx)])


def test_linear_one_hot_and_constant_inputs():
    """x = e_k picks column k of W_hat (pins nibble order and group addressing);
    a constant row per group sums the group's W_hat."""
    N, K = 9, 384
    W = _random_groups(N * K // 128, 21).reshape(N, K)
    st, qw, sc, z = oracle.quantize_pack(W)
    wh = oracle.dequant(qw, sc, z, K)
    codes = oracle.unpack(qw, K)
    for k in [0, 1, 7, 8, 127, 128, 255, 383]:
        X = np.zeros((1, K), dtype=np.uint16)
        X[0, k] = 0x3F80
        Y = oracle.linear(X, qw, sc, z)[0]
        g = k // 128
        expect = (codes[:, k].astype(np.float64) - z[:, g]) * oracle.bf16_to_f64(sc[:, g])
        np.testing.assert_array_equal(Y, expect)
        np.testing.assert_array_equal(Y, wh[:, k])
    X = np.zeros((1, K), dtype=np.uint16)
    X[0, 128:256] = 0x4000  # 2.0 on group 1 only
    Y = oracle.linear(X, qw, sc, z)[0]
    np.testing.assert_allclose(Y, 2.0 * wh[:, 128:256].sum(axis=1), rtol=1e-15, atol=0)


def test_dequant_bf16_is_rounded_exact_value():
    N, K = 16, 256
    W = _random_groups(N * K // 128, 31).reshape(N, K)
    st, qw, sc, z = oracle.quantize_pack(W)
    wh = oracle.dequant(qw, sc, z, K)
    lib_bits = torch.from_numpy(wh.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    # (q - z) * s has <= 13 significant bits, so the float32 cast is exact and torch's RNE applies
    np.testing.assert_array_equal(oracle.dequant_bf16(qw, sc, z, K), lib_bits)


def test_renorm_closed_forms():
    y = np.array([[0x4040, 0x4040, 0x4040, 0x4040],      # 3,3,3,3 -> all 1
                  [0x4040, 0x4080, 0x0000, 0x0000],      # 3,4,0,0 -> rms 2.5 -> 1.2, 1.6
                  [0x0000, 0x0000, 0x0000, 0x0000],      # zero row stays zero
                  [0xC040, 0x4040, 0xC040, 0x4040]], dtype=np.uint16)
    out, exact = oracle.renorm(y)
    np.testing.assert_array_equal(out[0], [0x3F80] * 4)
    np.testing.assert_allclose(exact[1], [1.2, 1.6, 0, 0], rtol=1e-15)
    np.testing.assert_array_equal(out[2], [0] * 4)
    np.testing.assert_array_equal(out[3], [0xBF80, 0x3F80, 0xBF80, 0x3F80])
    rng = np.random.default_rng(0)
    yb = torch.from_numpy(rng.standard_normal((3, 1000)).astype(np.float32) * 7).to(torch.bfloat16)
    out, exact = oracle.renorm(yb.view(torch.int16).numpy().view(np.uint16))
    np.testing.assert_allclose((exact ** 2).mean(axis=1), 1.0, rtol=1e-14)
