"""The SwiGLU kernel's rounding method, checked on the CPU (no GPU code runs).

The fused SwiGLU + requantization kernel must produce h = the correctly
rounded bf16 of g / (1 + exp(-g)) * u.  It evaluates the expression in FP32,
brackets the result by (1 -+ 2^-20) -- wider than the evaluation's error
bound, below 2.5 * 2^-22 with the exp and the quotient each within 2 ulp
(expf; div.full.f32) -- and keeps the bf16 both ends round to; otherwise it
evaluates in double and rounds to bf16 through round-to-odd FP32.  These
tests restate both steps with numpy, with the exp and the quotient each moved
by a random whole number of ulps in [-2, 2] (the device's worst cases lie in
that range), and check them against exact rounding of the real value.
"""
import math
from fractions import Fraction

import numpy as np

from workloads import bf16_bits, bf16_to_f32


def exact_bf16(v: float) -> int:
    """Round-to-nearest-even of a double to bf16 bits, by rational arithmetic."""
    if v == 0.0:
        return 0x8000 if math.copysign(1.0, v) < 0 else 0
    if math.isinf(v):
        return 0xFF80 if v < 0 else 0x7F80
    a = Fraction(abs(v))
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    ulp = Fraction(2) ** (e - 7) if e >= -126 else Fraction(2) ** -133
    n, rem = divmod(a, ulp)
    if rem * 2 > ulp or (rem * 2 == ulp and n % 2 == 1):
        n += 1
    y = n * ulp
    sign = 0x8000 if v < 0 else 0
    if y >= Fraction(2) ** 128:
        return sign | 0x7F80
    return sign | int(bf16_bits(np.array([float(y)], dtype=np.float32))[0])


def near_midpoint(v: float, rel: float = 1e-12) -> bool:
    """True when v is within rel of a bf16 rounding midpoint (where the double
    evaluation itself could not decide the rounding)."""
    if v == 0.0 or not math.isfinite(v):
        return False
    lo = float(bf16_to_f32(np.array([exact_bf16(v) & 0xFFFF], dtype=np.uint16))[0])
    m, e = math.frexp(abs(v))
    half_ulp = 2.0 ** (max(e - 1, -126) - 8)
    return min(abs(abs(v) - (abs(lo) + half_ulp)), abs(abs(v) - (abs(lo) - half_ulp))) <= rel * abs(v)


def ulp_shift(x: np.ndarray, k: np.ndarray) -> np.ndarray:
    """x moved by k (|k| <= 2) units in the last place, binary32."""
    x = x.astype(np.float32).copy()
    with np.errstate(over="ignore", invalid="ignore"):
        for step in (1, 2):
            up, dn = k >= step, k <= -step
            x[up] = np.nextafter(x[up], np.float32(np.inf), dtype=np.float32)
            x[dn] = np.nextafter(x[dn], np.float32(-np.inf), dtype=np.float32)
    return x


def fast_path(g: np.ndarray, u: np.ndarray, rng=None):
    """FP32 evaluation and the bracket test; returns (bf16 bits, decided mask).
    With rng, the exp and the quotient are each moved by up to 2 ulp."""
    with np.errstate(over="ignore", under="ignore", invalid="ignore", divide="ignore"):
        e = np.exp(-g).astype(np.float32)
        if rng is not None:
            e = ulp_shift(e, rng.integers(-2, 3, e.size))
        q = (g / (np.float32(1.0) + e)).astype(np.float32)
        if rng is not None:
            q = ulp_shift(q, rng.integers(-2, 3, q.size))
        h = (q * u).astype(np.float32)
        lo = (h * np.float32(1.0 - 2.0 ** -20)).astype(np.float32)
        hi = (h * np.float32(1.0 + 2.0 ** -20)).astype(np.float32)
    a = np.abs(h)
    ok = np.isfinite(e) & (a >= np.float32(2.0 ** -100)) & (a <= np.float32(2.0 ** 120))
    bl, bh = bf16_bits(np.where(ok, lo, 0)), bf16_bits(np.where(ok, hi, 0))
    return bl, ok & (bl == bh)


def test_fast_path_is_correctly_rounded():
    rng = np.random.default_rng(0)
    n = 200_000
    # GEMM1 outputs: gates of a few units, wide range of up values, some far gates
    g = bf16_to_f32(bf16_bits((rng.standard_normal(n) * np.exp(rng.uniform(-6, 3, n))).astype(np.float32)))
    u = bf16_to_f32(bf16_bits((rng.standard_normal(n) * np.exp(rng.uniform(-6, 5, n))).astype(np.float32)))
    bits, decided = fast_path(g, u, rng=np.random.default_rng(7))
    idx = np.flatnonzero(decided)
    assert decided.mean() > 0.998          # the double path is rare
    for i in idx[:: max(1, idx.size // 20000)]:
        gd, ud = float(g[i]), float(u[i])
        v = gd / (1.0 + math.exp(-gd)) * ud
        if near_midpoint(v):
            continue
        assert int(bits[i]) == exact_bf16(v), (gd, ud)


def test_fast_path_declines_outside_its_range():
    g = np.array([-89.0, -100.0, 0.0, 1e-30, 3e38, -3e38], dtype=np.float32)
    u = np.array([1.0, 1.0, 5.0, 1e-30, 2.0, 2.0], dtype=np.float32)
    _, decided = fast_path(g, u)
    # exp overflows, zero result, tiny result, product overflow: all take the double path
    assert not decided.any()


def round_to_odd_f32(v: float) -> np.float32:
    """Toward-zero conversion to binary32, then the last bit set if inexact."""
    with np.errstate(over="ignore"):
        f = np.float32(v)
    if math.isfinite(v) and abs(float(f)) > abs(v):
        f = np.nextafter(f, np.float32(0.0), dtype=np.float32)
    if math.isfinite(v) and abs(v) > float(np.finfo(np.float32).max):
        f = np.float32(math.copysign(float(np.finfo(np.float32).max), v))
    if math.isfinite(v) and float(f) != v:
        f = np.frombuffer(np.array([np.frombuffer(f.tobytes(), np.uint32)[0] | 1], np.uint32).tobytes(),
                          np.float32)[0]
    return f


def test_round_to_odd_then_bf16_rounds_once():
    """Double -> round-to-odd binary32 -> RNE bf16 equals RNE of the double
    directly, midpoints, subnormals and overflow included."""
    rng = np.random.default_rng(1)
    vals = list(rng.standard_normal(2000) * np.exp(rng.uniform(-90, 88, 2000)))
    # doubles just around bf16 midpoints: 1 + 2^-8 (a tie), and a hair either side
    for base in (1.0, 3.0, 2.0 ** -126, 2.0 ** -130, 2.0 ** 127):
        mid = base * (1 + 2.0 ** -8)
        vals += [mid, math.nextafter(mid, 0), math.nextafter(mid, math.inf), -mid]
    vals += [3.3961e38, 3.3962e38, 3.40e38, 1e39, -1e39, 5e-42, -5e-42]
    for v in vals:
        f = round_to_odd_f32(float(v))
        assert int(bf16_bits(np.array([f], dtype=np.float32))[0]) == exact_bf16(float(v)), v
