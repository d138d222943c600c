"""Comparison helpers shared by the GPU parity tests, smoke() and bench.py.

GEMM tolerance.  The target bounds the GEMM's error against the oracle's
dequantized-input product by a max relative error of 2e-3 and a max absolute
error of 1e-2 * rms(C).  The GEMM's result is delivered in bf16, whose unit
roundoff is 2^-8: rounding alone can move an element by up to
2^-8 / (1 + 2^-8) = 3.89e-3 relative, so the bound, applied literally to the
bf16 output, would reject even an exact computation.  The reading used here
applies the bound to the product *before* its one rounding to bf16:

  every output element C must be the round-to-nearest-even bf16 of some value
  v with |v - C_ref| <= d, where
      d = min(2e-3 * |C_ref|, 1e-2 * rms(C_ref))   if |C_ref| >= 0.1 * rms(C_ref)
      d = 1e-2 * rms(C_ref)                          otherwise
  (relative error is meaningless for near-zero elements, which cancellation
  produces; they are held to the absolute bound).

Equivalently the implied pre-rounding error e = distance from C_ref to the set
of reals that round to C must satisfy e <= d.  The statistics also report the
raw output error and how many elements are not the correctly rounded C_ref.
"""
from __future__ import annotations

import numpy as np
import torch

REL_TOL = 2e-3
ABS_TOL_RMS = 1e-2
REL_FLOOR_RMS = 0.1


def to_torch_bf16(bits: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def bf16_bits_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bytes_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.uint8).cpu().numpy()


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    # a signalling-NaN pattern raises the invalid flag in the widening; it stays a NaN
    with np.errstate(invalid="ignore"):
        return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_rne_f64(x: np.ndarray) -> np.ndarray:
    """float64 -> nearest bf16 value (ties to even), one rounding, as float64.
    (Normal range only; the magnitudes compared here are far from bf16's
    subnormals.)"""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)  # x = m * 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0), e - 8)  # 8 significant bits, rint = half-to-even


def _neighbours(bits: np.ndarray):
    """bf16 values just above and just below each pattern (as float64)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.int32)
    mag = b & 0x7FFF
    neg = (b & 0x8000) != 0
    up_bits = np.where(neg, np.where(mag > 0, 0x8000 | (mag - 1), 0x0001), mag + 1)
    dn_bits = np.where(neg, 0x8000 | (mag + 1), np.where(mag > 0, mag - 1, 0x8001))
    return bf16_to_f64(up_bits.astype(np.uint16)), bf16_to_f64(dn_bits.astype(np.uint16))


def gemm_errors(c_bits: np.ndarray, ref: np.ndarray) -> dict:
    c = bf16_to_f64(c_bits)
    ref = np.asarray(ref, dtype=np.float64)
    assert c.shape == ref.shape, (c.shape, ref.shape)
    n = ref.size
    rms = float(np.sqrt(np.mean(ref * ref))) if n else 0.0
    big = np.abs(ref) >= REL_FLOOR_RMS * rms
    d = np.full(ref.shape, ABS_TOL_RMS * rms)
    d[big] = np.minimum(d[big], REL_TOL * np.abs(ref[big]))
    up, dn = _neighbours(c_bits)
    half_up = (up - c) / 2.0
    half_dn = (c - dn) / 2.0
    implied = np.where(ref > c, np.maximum(0.0, ref - c - half_up), np.maximum(0.0, c - ref - half_dn))
    err = np.abs(c - ref)
    finite = np.isfinite(c)
    with np.errstate(divide="ignore", invalid="ignore"):
        used = np.where(d > 0, implied / d, np.where(implied > 0, np.inf, 0.0))
    return {
        "rms": rms,
        "n": int(n),
        "n_rel": int(big.sum()),
        "tol_used": float(used.max()) if n else 0.0,             # <= 1 passes
        "implied_max_rel": float((implied[big] / np.abs(ref[big])).max()) if big.any() else 0.0,
        "implied_max_abs_over_rms": float(implied.max() / rms) if n and rms > 0 else 0.0,
        "out_max_rel": float((err[big] / np.abs(ref[big])).max()) if big.any() else 0.0,
        "out_max_abs_over_rms": float(err.max() / rms) if n and rms > 0 else 0.0,
        "not_correctly_rounded": int(np.count_nonzero(c != bf16_rne_f64(ref))),
        "nonfinite": int(np.count_nonzero(~finite)),
    }


def gemm_ok(stats: dict) -> bool:
    return stats["nonfinite"] == 0 and stats["tol_used"] <= 1.0


def assert_gemm_close(c_bits: np.ndarray, ref: np.ndarray, what: str = "gemm") -> dict:
    st = gemm_errors(c_bits, ref)
    assert gemm_ok(st), "%s outside tolerance: %s" % (what, st)
    return st
