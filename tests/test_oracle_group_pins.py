"""Pins for the oracle's smaller quantisation groups (32 and 64 consecutive weights
along K: "Quantization I: int8, int4, the basics", Concept, groups of 32-128 values;
"Weight-Only Quantization and Mixed Precision", section 8, group size 32/64/128),
with the model card's per-group rule unchanged.  Expected values come from closed
forms, grid round trips, the independently pinned group-128 quantiser and numpy's
FP64 matmul -- never from the group-32/64 code under test.
"""
import numpy as np
import pytest

import oracle

S7 = 2.0 ** -7


@pytest.mark.parametrize("G", [32, 64])
def test_handworked_groups_with_their_own_zero_points(G):
    """Group j holds ((k mod 16) - z_j) 2^-7: s = 2^-7, z = z_j, q = k mod 16 in every group."""
    K = 256
    zs = [5, 3, 0, 7, 12, 1, 9, 4][: K // G]
    k = np.arange(K)
    w = ((k % 16) - np.repeat(zs, G)) * S7
    st, qw, sc, z = oracle.quantize_pack_g(w[None, :], G)
    assert st == oracle.OK
    np.testing.assert_array_equal(sc[0], np.full(K // G, 0x3C00))
    np.testing.assert_array_equal(z[0], zs)
    np.testing.assert_array_equal(qw[0], np.tile([0x76543210, 0xFEDCBA98], K // 16))
    np.testing.assert_array_equal(oracle.dequant_g(qw, sc, z, K)[0], w)


@pytest.mark.parametrize("G", [32, 64])
def test_requantize_grid_aligned(G):
    rng = np.random.default_rng(80 + G)
    N, K = 300, 512
    codes = rng.integers(0, 16, size=(N, K // G, G))
    codes[:, :, 0] = 0
    codes[:, :, 1] = 15
    zs = rng.integers(-20, 36, size=(N, K // G))
    sbits = rng.integers(0x3A00, 0x3E00, size=(N, K // G)).astype(np.uint16)
    s = oracle.bf16_to_f64(sbits)
    W = ((codes - zs[:, :, None]) * s[:, :, None]).reshape(N, K).astype(np.float32)
    st, qw, sc, z = oracle.quantize_pack_g(W, G)
    assert st == oracle.OK
    np.testing.assert_array_equal(sc, sbits)
    np.testing.assert_array_equal(z, zs)
    np.testing.assert_array_equal(oracle.unpack(qw, K), codes.reshape(N, K))


@pytest.mark.parametrize("G", [32, 64])
def test_smaller_groups_stay_within_the_group128_step(G):
    """A sub-group's range is at most its 128-group's, so its scale is at most the group-128
    scale and every unclipped weight is within half that step; the error shrinks on average."""
    rng = np.random.default_rng(90 + G)
    W = (rng.standard_normal((400, 1024)) * 0.02).astype(np.float32)
    W[::3, ::97] *= 8.0
    st, qw, sc, z, cl = oracle.quantize_pack_g(W, G, with_clipped=True)
    st128, qw128, sc128, z128 = oracle.quantize_pack(W)
    assert st == st128 == oracle.OK
    s128 = np.repeat(oracle.bf16_to_f64(sc128), 128, axis=1)
    err = np.abs(oracle.dequant_g(qw, sc, z, 1024) - W.astype(np.float64))
    ok = cl == 0
    assert np.all(err[ok] <= s128[ok] / 2)
    err128 = np.abs(oracle.dequant(qw128, sc128, z128, 1024) - W.astype(np.float64))
    assert err.mean() < err128.mean()


@pytest.mark.parametrize("G", [32, 64])
def test_linear_matches_library_matmul_and_one_hot(G):
    rng = np.random.default_rng(100 + G)
    M, N, K = 5, 48, 384
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    st, qw, sc, z = oracle.quantize_pack_g(W, G)
    xbits = (rng.standard_normal((M, K)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    wh = oracle.dequant_g(qw, sc, z, K)
    want = oracle.bf16_to_f64(xbits) @ wh.T
    np.testing.assert_allclose(oracle.linear_g(xbits, qw, sc, z), want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    onehot = np.zeros((3, K), dtype=np.uint16)
    for i, k in enumerate([0, G - 1, G + 5]):
        onehot[i, k] = 0x3F80
    got = oracle.linear_g(onehot, qw, sc, z)
    for i, k in enumerate([0, G - 1, G + 5]):
        np.testing.assert_array_equal(got[i], wh[:, k])


def test_group128_entry_agrees_and_metadata_cost():
    """The _g entry with G = 128 is the format's quantiser; bits per weight are 4 + 48 / G
    (a BF16 scale and an INT32 zero point per group: more metadata for smaller groups)."""
    rng = np.random.default_rng(111)
    W = (rng.standard_normal((64, 512)) * 0.02).astype(np.float32)
    a = oracle.quantize_pack_g(W, 128)
    b = oracle.quantize_pack(W)
    for x, y in zip(a[1:], b[1:]):
        np.testing.assert_array_equal(x, y)
    for G, bits in [(32, 5.5), (64, 4.75), (128, 4.375)]:
        assert 4 + (2 + 4) * 8 / G == bits
    st, *_ = oracle.quantize_pack_g(W, 48)
    assert st == oracle.ERR_ARG


def test_symmetric_small_groups():
    rng = np.random.default_rng(112)
    W = (rng.standard_normal((32, 256)) * 0.02).astype(np.float32)
    st, qw, sc, z = oracle.quantize_pack_g(W, 32, symmetric=True)
    assert st == oracle.OK and np.all(z == 8)
    s = np.repeat(oracle.bf16_to_f64(sc), 32, axis=1)
    q = oracle.unpack(qw, 256).astype(np.float64) - 8
    assert np.all(np.abs(q * s - W) <= s / 2)
