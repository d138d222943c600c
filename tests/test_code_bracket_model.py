"""The quantizers' division-free code method, replayed on the CPU (no GPU code runs).

The kernels produce E4M3(fl32(x / s)) without dividing on the common path:
two products x * r_lo and x * r_hi with r_lo < 1/s < r_hi (the bracket checked
exactly with FMA residuals) give an element's code when both round to the same
code; an element whose two codes differ is recomputed from the IEEE quotient,
alone.  These tests restate the method with numpy -- float32 products and
residuals evaluated exactly in float64, then rounded once -- with the bracket
built around fl32(1/s) instead of the hardware's approximate reciprocal (the
exact check makes the source of the approximation irrelevant), and compare its
codes with the oracle's.  They also measure how often the two codes differ on
bf16 data and show why: mostly exact E4M3 ties of 448 x / amax.
"""
from fractions import Fraction

import numpy as np

import oracle
from workloads import bf16_bits, bf16_to_f32

WIDEN = 2.0 ** -20


def f32_mul(a, b):
    """fl32(a * b) for float32 operands: the float64 product is exact (48 bits)."""
    return (a.astype(np.float64) * b.astype(np.float64)).astype(np.float32)


MIN_FAST_SCALE = np.float32(2.0 ** -125)   # below it a group takes the division path whole


def bracket(s):
    """r_lo, r_hi around 1/s and whether the exact residual checks hold
    (groups with s below MIN_FAST_SCALE are not bracketed)."""
    s = np.maximum(s, MIN_FAST_SCALE)
    r = (1.0 / s.astype(np.float64)).astype(np.float32)
    lo = f32_mul(r, np.float32(1.0 - WIDEN) + np.zeros_like(r))
    hi = f32_mul(r, np.float32(1.0 + WIDEN) + np.zeros_like(r))
    # 1 - s * r is exact in float64 (s * r has 48 bits and lies near 1)
    ok = (1.0 - s.astype(np.float64) * lo > 0) & (1.0 - s.astype(np.float64) * hi < 0)
    return lo, hi, ok


def codes_by_method(x, s):
    """x [G, 128] float32, s [G] float32 -> (codes, mask of elements that took the division)."""
    lo, hi, ok = bracket(s)
    assert ok.all()
    whole = (s < MIN_FAST_SCALE)[:, None]
    c_lo = oracle.e4m3_encode_array(f32_mul(x, lo[:, None]))
    c_hi = oracle.e4m3_encode_array(f32_mul(x, hi[:, None]))
    split = (c_lo != c_hi) | whole
    q = (x / s[:, None]).astype(np.float32)          # IEEE binary32 quotient
    codes = np.where(split, oracle.e4m3_encode_array(q), c_lo)
    return codes.astype(np.uint8), split


def groups_of(bits):
    """bf16 bits [M, K] -> x [M*K/128, 128] float32 and the oracle's codes and scales."""
    q, s = oracle.quant_act_1x128(bits)
    x = bf16_to_f32(bits).reshape(-1, 128).astype(np.float32)
    return x, q.reshape(-1, 128), s.reshape(-1).astype(np.float32)


def test_method_matches_the_oracle_on_normal_data():
    rng = np.random.default_rng(11)
    bits = bf16_bits(rng.standard_normal((256, 2048)).astype(np.float32))
    x, q, s = groups_of(bits)
    codes, split = codes_by_method(x, s)
    assert np.array_equal(codes, q)
    assert split.any()


def test_method_matches_the_oracle_for_every_16th_bf16_amax():
    amax = bf16_to_f32(np.arange(16, 0x7F80, 16, dtype=np.uint16)).astype(np.float32)
    rng = np.random.default_rng(12)
    x = amax[:, None] * rng.uniform(-1.0, 1.0, (amax.size, 128)).astype(np.float32)
    x[:, 5] = amax
    bits = bf16_bits(x.astype(np.float32))
    xg, q, s = groups_of(bits.reshape(-1, 128))
    codes, _ = codes_by_method(xg, s)
    assert np.array_equal(codes, q)


def test_split_codes_are_common_and_are_exact_ties():
    """About 0.5% of normally distributed bf16 elements get two different
    bracket codes, and every one is a quotient 448 x / amax lying exactly on an
    E4M3 rounding midpoint.  x and amax both have 8-bit significands, so a
    quotient that is not a tie is at least ~2^-13 (relative) from any midpoint,
    far outside the 2^-20 bracket; a tie stays within 2^-24 of its midpoint
    after s = fl32(amax / 448) is rounded."""
    rng = np.random.default_rng(13)
    bits = bf16_bits(rng.standard_normal((512, 2048)).astype(np.float32))
    x, _, s = groups_of(bits)
    _, split = codes_by_method(x, s)
    rate = split.mean()
    assert 0.003 < rate < 0.008, rate
    amax = np.abs(x).max(axis=1)
    mids = sorted({Fraction(float(oracle.e4m3_decode(c))) for c in range(0x7F)})
    mids = {(a + b) / 2 for a, b in zip(mids[:-1], mids[1:])}
    rows, cols = np.nonzero(split)
    assert all(Fraction(abs(float(x[r, c]))) * 448 / Fraction(float(amax[r])) in mids for r, c in zip(rows, cols))
