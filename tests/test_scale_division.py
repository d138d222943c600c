"""The quantizers' division-free group scale, checked exhaustively on the host.

The scale of a group is s = fl32(amax / 448) (IEEE division).  The kernels
compute it as
    q0 = RN(amax * c),  r = RN(amax - 448 q0),  s = RN(q0 + r c),  c = RN(1/448)
(one multiply, two fused multiply-adds).  amax is a bf16 magnitude, so there
are only 32640 finite non-negative inputs; this test replays the sequence in
exact rational arithmetic with one binary32 rounding per operation (what a
fused multiply-add does) and requires the correctly rounded quotient for every
one of them, subnormal results included.  The GPU side is covered by the
every-amax parity test against the oracle.
"""
from fractions import Fraction

import numpy as np

SMALLEST = Fraction(1, 2 ** 149)  # binary32 subnormal spacing


def rn32(x: Fraction) -> Fraction:
    """Round a rational to binary32 (nearest, ties to even), finite range."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    ulp = Fraction(2) ** (e - 23) if e >= -126 else SMALLEST
    n, rem = divmod(a, ulp)
    if rem * 2 > ulp or (rem * 2 == ulp and n % 2 == 1):
        n += 1
    return sign * n * ulp


def test_rn32_matches_numpy_on_samples():
    rng = np.random.default_rng(0)
    for v in rng.standard_normal(200) * np.exp(rng.uniform(-80, 80, 200)):
        assert rn32(Fraction(float(v))) == Fraction(float(np.float32(v)))


def test_scale_sequence_is_the_correctly_rounded_quotient():
    c = rn32(Fraction(1, 448))
    assert c == Fraction(float(np.float32(1) / np.float32(448)))
    bits = np.arange(0, 0x7F80, dtype=np.uint32) << 16  # every finite non-negative bf16
    values = bits.view(np.float32)
    bad = []
    for a32 in values:
        a = Fraction(float(a32))
        want = rn32(a / 448)
        q0 = rn32(a * c)
        r = rn32(a - 448 * q0)
        got = rn32(q0 + r * c)
        if got != want:
            bad.append(float(a32))
    assert not bad, bad[:5]


def test_single_product_is_not_enough():
    """The correction step matters: RN(amax * c) alone misses about half."""
    c = rn32(Fraction(1, 448))
    misses = 0
    for m in range(128, 256):  # one binade of 8-bit significands
        a = Fraction(m, 128)
        misses += rn32(a * c) != rn32(a / 448)
    assert misses > 0
