"""Seeded activations with extreme per-group dynamic range, as BF16 bit patterns.

The decode kernels re-express every group of 128 activations as integers
relative to the group's largest magnitude, so the inputs that stress them are
groups whose values span many binades, exact zeros, all-zero groups, negative
maxima, BF16 subnormals, and magnitudes near both ends of the BF16 range.
Each token row takes one kind for all of its groups, so a row's outputs can be
compared under a tolerance scaled to that row alone.

Values are built directly as bit patterns (sign, exponent field, 7 mantissa
bits) from numpy's seeded generator; nothing here computes any part of the
linear layer.  Shared by the parity tests only.
"""
from __future__ import annotations

import numpy as np

GROUP = 128
BF16_MAX_FINITE = 0x7F7F   # (2 - 2^-7) * 2^127
BF16_ONE_TWO10 = 0x4480    # 2^10

KINDS = (
    "control",          # exponents in [-6, 2): ordinary activations
    "wide",             # one +-2^10 per group beside magnitudes down to 2^-10 (20 binades below it)
    "wide_zeros",       # as wide, about half the values exactly +0 or -0
    "zero_groups",      # every other group all zero (+0 and -0), the rest ordinary
    "neg_max",          # each group's largest magnitude is a negative value (-8 .. -16)
    "subnormal",        # every value a BF16 subnormal or zero
    "subnormal_mixed",  # subnormals beside ordinary values in every group
    "tiny",             # smallest normal binades: exponents in [-126, -116)
    "huge",             # exponents in [90, 100)
    "max_finite",       # one +-largest finite BF16 in the first group, the rest ordinary
    "zero_row",         # every value +0 or -0
)


def _bits(rng, n, e_lo, e_hi):
    """n random normal BF16 patterns with unbiased exponent in [e_lo, e_hi) and random signs."""
    e = rng.integers(e_lo + 127, e_hi + 127, size=n)
    m = rng.integers(0, 128, size=n)
    s = rng.integers(0, 2, size=n)
    return ((s << 15) | (e << 7) | m).astype(np.uint16)


def _subnormal_bits(rng, n):
    m = rng.integers(0, 128, size=n)  # 0 gives a (signed) zero
    s = rng.integers(0, 2, size=n)
    return ((s << 15) | m).astype(np.uint16)


def _zero_bits(rng, n):
    return (rng.integers(0, 2, size=n) << 15).astype(np.uint16)


def _row(rng, kind: str, K: int) -> np.ndarray:
    G = K // GROUP
    row = np.empty(K, dtype=np.uint16)
    for g in range(G):
        sl = slice(g * GROUP, (g + 1) * GROUP)
        if kind == "control":
            v = _bits(rng, GROUP, -6, 2)
        elif kind in ("wide", "wide_zeros"):
            v = _bits(rng, GROUP, -10, 10)
            if kind == "wide_zeros":
                z = rng.random(GROUP) < 0.5
                v[z] = _zero_bits(rng, int(z.sum()))
            v[rng.integers(0, GROUP)] = BF16_ONE_TWO10 | (int(rng.integers(0, 2)) << 15)
        elif kind == "zero_groups":
            v = _zero_bits(rng, GROUP) if g % 2 == 0 else _bits(rng, GROUP, -6, 2)
        elif kind == "neg_max":
            v = _bits(rng, GROUP, -6, 2)
            v[rng.integers(0, GROUP)] = 0x8000 | ((3 + 127) << 7) | int(rng.integers(0, 128))
        elif kind == "subnormal":
            v = _subnormal_bits(rng, GROUP)
        elif kind == "subnormal_mixed":
            v = _bits(rng, GROUP, -4, 2)
            sub = rng.random(GROUP) < 0.5
            v[sub] = _subnormal_bits(rng, int(sub.sum()))
        elif kind == "tiny":
            v = _bits(rng, GROUP, -126, -116)
        elif kind == "huge":
            v = _bits(rng, GROUP, 90, 100)
        elif kind == "max_finite":
            v = _bits(rng, GROUP, -4, 2)
            if g == 0:
                v[rng.integers(0, GROUP)] = BF16_MAX_FINITE | (int(rng.integers(0, 2)) << 15)
        elif kind == "zero_row":
            v = _zero_bits(rng, GROUP)
        else:
            raise ValueError(f"unknown kind {kind}")
        row[sl] = v
    return row


def activations_bf16(seed: int, kinds, K: int) -> np.ndarray:
    """X [len(kinds), K] as BF16 bit patterns; row m is of kind kinds[m]."""
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    rng = np.random.default_rng(seed)
    return np.stack([_row(rng, k, K) for k in kinds]).astype(np.uint16)
