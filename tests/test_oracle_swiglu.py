"""Pins for the oracle's SwiGLU step between the two MoE GEMMs (CPU only).

The step is not on the pages; the configurations imply it (GEMM1's N = 4096
is twice GEMM2's K = 2048).  Reading: each GEMM1 output row is [gate | up],
h = silu(gate) * up with silu(g) = g / (1 + exp(-g)), computed in double and
rounded once to bf16 (round to nearest, ties to even).
"""
import math
from fractions import Fraction

import numpy as np
import pytest

from workloads import bf16_bits, bf16_to_f32


def _rne_bf16(v: float) -> float:
    """Exact round-to-nearest-even of a double to bf16 (8 significant bits), by rational arithmetic."""
    if v == 0.0 or not math.isfinite(v):
        return v
    a = Fraction(abs(v))
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    ulp = Fraction(2) ** (e - 7) if e >= -126 else Fraction(2) ** -133
    n, rem = divmod(a, ulp)
    if rem * 2 > ulp or (rem * 2 == ulp and n % 2 == 1):
        n += 1
    return math.copysign(float(n * ulp), v)


def _bits(values):
    return bf16_bits(np.asarray(values, dtype=np.float32))


def _run(orc, gate, up):
    c1 = np.concatenate([_bits(gate), _bits(up)], axis=-1)
    return bf16_to_f32(orc.swiglu_bf16(c1))


def test_zero_gate_or_up_gives_zero(orc):
    h = _run(orc, [[0.0, 0.0, 3.0, -3.0]], [[5.0, -7.0, 0.0, 0.0]])
    assert np.all(h == 0.0)


def test_closed_forms(orc):
    # silu(1) * 1 = 1 / (1 + e^-1); silu(100) = 100 to double precision; silu(-100) ~ -3.7e-42 -> -0
    h = _run(orc, [[1.0, 100.0, -100.0, 2.0]], [[1.0, 3.0, 1.0, -0.5]])
    assert h[0, 0] == _rne_bf16(1.0 / (1.0 + math.exp(-1.0)))
    assert h[0, 1] == 300.0
    assert h[0, 2] == 0.0 and math.copysign(1.0, h[0, 2]) == -1.0  # underflows, sign kept
    assert h[0, 3] == _rne_bf16(2.0 / (1.0 + math.exp(-2.0)) * -0.5)


def test_silu_odd_part_identity(orc):
    """silu(x) - silu(-x) = x: the two outputs differ by x up to their two bf16 roundings."""
    x = bf16_to_f32(_bits(np.linspace(-8, 8, 97)))
    hp = _run(orc, x[None, :], np.ones((1, x.size)))[0]
    hm = _run(orc, -x[None, :], np.ones((1, x.size)))[0]
    tol = 2.0 ** -8 * (np.abs(hp) + np.abs(hm)) + 1e-30
    assert np.all(np.abs((hp - hm) - x) <= tol)


def test_random_rows_match_exact_rounding(orc):
    rng = np.random.default_rng(40)
    rows, inter = 6, 256
    c1 = bf16_bits((3 * rng.standard_normal((rows, 2 * inter))).astype(np.float32))
    h = bf16_to_f32(orc.swiglu_bf16(c1))
    g = bf16_to_f32(c1[:, :inter]).astype(np.float64)
    u = bf16_to_f32(c1[:, inter:]).astype(np.float64)
    exact = g / (1.0 + np.exp(-g)) * u
    expect = np.vectorize(_rne_bf16)(exact)
    assert np.array_equal(h.astype(np.float64), expect)


def test_batched_shape(orc):
    rng = np.random.default_rng(41)
    c1 = bf16_bits(rng.standard_normal((2, 3, 256)).astype(np.float32))
    h = orc.swiglu_bf16(c1)
    assert h.shape == (2, 3, 128)
    assert np.array_equal(h.reshape(6, 128), orc.swiglu_bf16(c1.reshape(6, 256)))
    with pytest.raises(ValueError):
        orc.swiglu_bf16(c1[..., :255])


def test_round_bf16_matches_exact_rounding(orc):
    rng = np.random.default_rng(42)
    v = rng.standard_normal(500) * np.exp(rng.uniform(-60, 60, 500))
    v[:4] = [0.0, -0.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8]  # ties: to 1.0 and to 1 + 2^-6
    got = bf16_to_f32(orc.round_bf16(v)).astype(np.float64)
    assert np.array_equal(got, np.vectorize(_rne_bf16)(v))
    assert got[2] == 1.0 and got[3] == 1.0 + 2.0 ** -6
    assert math.copysign(1.0, got[1]) == -1.0


def test_masked_chain_is_the_composition_of_its_steps(orc):
    """The chained decode equals its steps run one after another, and rows at
    or past each expert's count stay unwritten."""
    rng = np.random.default_rng(43)
    E, cap, K1, inter, N2 = 3, 128, 256, 128, 256
    a = bf16_bits(rng.standard_normal((E, cap, K1)).astype(np.float32))
    b1 = bf16_bits((0.05 * rng.standard_normal((E, 2 * inter, K1))).astype(np.float32))
    b2 = bf16_bits((0.05 * rng.standard_normal((E, N2, inter))).astype(np.float32))
    mm = np.array([0, 5, 128], dtype=np.int32)
    out = orc.masked_moe_chain(a, b1, b2, mm)
    assert out.shape == (E, cap, N2)
    assert np.all(np.isnan(out[0])) and np.all(np.isnan(out[1, 5:])) and not np.any(np.isnan(out[2]))
    # expert 2, row 7, by hand from the steps
    qa, sa = orc.quant_act_1x128(a[2])
    qb1, sb1 = orc.quant_w_128x128(b1[2])
    c1 = orc.gemm_blockscaled(qa, sa, qb1, sb1, rows=[7])
    h = orc.swiglu_bf16(orc.round_bf16(c1))
    qh_all, sh_all = orc.quant_act_1x128(orc.swiglu_bf16(orc.round_bf16(orc.gemm_blockscaled(qa, sa, qb1, sb1))))
    assert np.array_equal(qh_all[7:8], orc.quant_act_1x128(h)[0])
    qb2, sb2 = orc.quant_w_128x128(b2[2])
    row = orc.gemm_blockscaled(qh_all, sh_all, qb2, sb2, rows=[7])
    assert np.array_equal(out[2, 7], row[0])
