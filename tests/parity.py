"""Comparison helpers shared by the GPU parity tests, smoke() and bench.py.

GEMM tolerance (the target's own wording: max relative error 2e-3 and max
absolute error <= 1e-2 * rms(C) against the oracle's dequantized-input
product).  Read as two checks over the compared elements:
  (1) max |C - C_ref| <= 1e-2 * rms(C_ref)
  (2) max |C - C_ref| / |C_ref| <= 2e-3 over elements with |C_ref| >= 0.1 * rms(C_ref)
(near-zero elements make a pure relative error meaningless).  bf16 rounding
of the output alone spends up to 2^-9 / (1 + 2^-9) = 1.949e-3 of (2).
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
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def gemm_errors(c_bits: np.ndarray, ref: np.ndarray) -> dict:
    """Error statistics of a bf16 result (bit patterns) against float64 ref."""
    c = bf16_to_f64(c_bits)
    ref = np.asarray(ref, dtype=np.float64)
    assert c.shape == ref.shape, (c.shape, ref.shape)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    err = np.abs(c - ref)
    big = np.abs(ref) >= REL_FLOOR_RMS * rms
    rel = err[big] / np.abs(ref[big]) if big.any() else np.zeros(1)
    ref_bf16 = torch.from_numpy(ref).to(torch.bfloat16).to(torch.float64).numpy()
    ulp = np.abs(ref_bf16) * 2.0 ** -7
    beyond_1ulp = int(np.count_nonzero(np.abs(c - ref_bf16) > np.maximum(ulp, 1e-30) * 1.0001))
    return {
        "rms": rms,
        "max_abs": float(err.max()) if err.size else 0.0,
        "max_abs_over_rms": float(err.max() / rms) if err.size and rms > 0 else 0.0,
        "max_rel": float(rel.max()),
        "n": int(ref.size),
        "n_rel": int(big.sum()),
        "beyond_1ulp": beyond_1ulp,
        "nonfinite": int(np.count_nonzero(~np.isfinite(c))),
    }


def gemm_ok(stats: dict) -> bool:
    return (stats["nonfinite"] == 0 and stats["max_abs_over_rms"] <= ABS_TOL_RMS and stats["max_rel"] <= REL_TOL)


def assert_gemm_close(c_bits: np.ndarray, ref: np.ndarray, what: str = "gemm") -> dict:
    st = gemm_errors(c_bits, ref)
    assert gemm_ok(st), "%s outside tolerance: %s" % (what, st)
    return st
