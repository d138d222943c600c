"""Scaling-accuracy study on the CPU oracle: fine-grained vs per-tensor vs delayed scaling.

TEST INFRASTRUCTURE ONLY (like the rest of ``oracle/``): it calls the oracle
and the seeded workload generators, nothing of the product library.

"The Insider Secrets Of Deepseek Discovered" (FP8 mixed-precision passage)
says that scaling a whole tensor by its largest magnitude lets a few outliers
push the other values toward FP8's underflow, and that 1x128 / 128x128 groups
contain that damage (Figure 7 (a)).  The codingmall DeepSeek-V3 FP8 page
contrasts its online scales (taken from the current values) with delayed
scaling, which takes the scale from earlier iterations' maxima.  This script
measures all three, plus the fine-grained groups with power-of-two (UE8M0)
scales, on the dense_fprop workload (per-channel log-normal
activations with +-200 outliers, N(0, 0.02) weights): the error of the
block-scaled product against the exact product of the unquantized bf16
inputs, on a seeded sample of rows.

Delayed scaling needs an amax history the pages do not give; two plain
histories are used, each stated in the output:
  * growing activations: the previous 16 steps had the same values scaled by
    0.98^age, so the history's maximum is 0.98 of the current amax;
  * a new outlier: one current activation is set to 4x the tensor's amax,
    which no earlier step had, so the history's maximum is the old amax.

Usage: python -m oracle.scaling_accuracy [--rows-step 16] [--workload dense_fprop]
"""
from __future__ import annotations

import argparse
import time

import numpy as np

from . import (TILE, e4m3_decode_table, gemm_blockscaled, quant_act_1x128, quant_act_1x128_ue8m0, quant_tensor,
               quant_w_128x128, quant_w_128x128_ue8m0, quant_with_scale)


def _f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _errors(c: np.ndarray, ref: np.ndarray) -> dict:
    rms = float(np.sqrt(np.mean(ref * ref)))
    big = np.abs(ref) >= 0.1 * rms
    rel = np.abs(c - ref)[big] / np.abs(ref)[big]
    return {"fro_rel": float(np.linalg.norm(c - ref) / np.linalg.norm(ref)),
            "max_rel": float(rel.max()) if rel.size else 0.0,
            "median_rel": float(np.median(rel)) if rel.size else 0.0}


def _dequant_rel_rms(x_bits: np.ndarray, q: np.ndarray, scales: np.ndarray) -> float:
    """Relative RMS error of the dequantized tensor (scales broadcast per element)."""
    dec = e4m3_decode_table()[q] * scales
    x = _f64(x_bits)
    return float(np.sqrt(np.mean((dec - x) ** 2)) / np.sqrt(np.mean(x * x)))


def _const_scales(s: float, rows: int, cols: int) -> np.ndarray:
    return np.full((rows, cols), s, dtype=np.float32)


def study(a_bits: np.ndarray, b_bits: np.ndarray, rows: np.ndarray) -> list[dict]:
    """One row per scheme: name, activation dequantization error, GEMM errors."""
    M, K = a_bits.shape
    N = b_bits.shape[0]
    nkb, nnb = K // TILE, N // TILE
    ref = _f64(a_bits[rows]) @ _f64(b_bits).T
    out = []

    # fine-grained, online (the method)
    qa, sa = quant_act_1x128(a_bits)
    qb, sb = quant_w_128x128(b_bits)
    out.append(dict(name="fine-grained 1x128 / 128x128, online",
                    act_err=_dequant_rel_rms(a_bits, qa, np.repeat(sa, TILE, axis=1)),
                    saturated=0, **_errors(gemm_blockscaled(qa, sa, qb, sb, rows), ref)))

    # fine-grained groups with power-of-two (UE8M0) scales, the microscaling variant
    qa2, sa2 = quant_act_1x128_ue8m0(a_bits)
    qb2, sb2 = quant_w_128x128_ue8m0(b_bits)
    out.append(dict(name="fine-grained 1x128 / 128x128, power-of-two (UE8M0) scales",
                    act_err=_dequant_rel_rms(a_bits, qa2, np.repeat(sa2, TILE, axis=1)),
                    saturated=0, **_errors(gemm_blockscaled(qa2, sa2, qb2, sb2, rows), ref)))

    # per-tensor, online
    qa_t, s_a = quant_tensor(a_bits)
    qb_t, s_b = quant_tensor(b_bits)
    sa_t, sb_t = _const_scales(s_a, M, nkb), _const_scales(s_b, nnb, nkb)
    out.append(dict(name="per-tensor, online",
                    act_err=_dequant_rel_rms(a_bits, qa_t, np.float64(s_a)),
                    saturated=0, **_errors(gemm_blockscaled(qa_t, sa_t, qb_t, sb_t, rows), ref)))

    amax = float(np.max(np.abs(_f64(a_bits))))

    # per-tensor, delayed: growing activations (history max = 0.98 amax)
    s_hist = np.float32(np.float32(0.98 * amax) / np.float32(448.0))
    qa_d = quant_with_scale(a_bits, s_hist)
    sat = int(np.count_nonzero(np.abs(_f64(a_bits)) > 448.0 * float(s_hist)))
    out.append(dict(name="per-tensor, delayed (history max 0.98 x current amax)",
                    act_err=_dequant_rel_rms(a_bits, qa_d, np.float64(s_hist)), saturated=sat,
                    **_errors(gemm_blockscaled(qa_d, _const_scales(s_hist, M, nkb), qb_t, sb_t, rows), ref)))

    # per-tensor, delayed: a new outlier at 4x the old amax in a sampled row
    spiked = a_bits.copy()
    r0, k0 = int(rows[0]), K // 3
    spiked[r0, k0] = (np.array([4.0 * amax], dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)[0]
    ref_s = _f64(spiked[rows]) @ _f64(b_bits).T
    s_old = np.float32(np.float32(amax) / np.float32(448.0))
    qa_s = quant_with_scale(spiked, s_old)
    qa_f, sa_f = quant_act_1x128(spiked)
    out.append(dict(name="per-tensor, delayed (new outlier at 4x the history max)",
                    act_err=_dequant_rel_rms(spiked, qa_s, np.float64(s_old)), saturated=1,
                    **_errors(gemm_blockscaled(qa_s, _const_scales(s_old, M, nkb), qb_t, sb_t, rows), ref_s)))
    out.append(dict(name="fine-grained, online, same new outlier",
                    act_err=_dequant_rel_rms(spiked, qa_f, np.repeat(sa_f, TILE, axis=1)), saturated=0,
                    **_errors(gemm_blockscaled(qa_f, sa_f, qb, sb, rows), ref_s)))
    return out


def table(results: list[dict]) -> str:
    lines = ["| scheme | activation dequant rel. RMS error | GEMM rel. Frobenius error | GEMM max rel. error "
             "(\\|C\\| >= 0.1 rms) | GEMM median rel. error | saturated activations |",
             "|---|---:|---:|---:|---:|---:|"]
    for r in results:
        lines.append("| %s | %.2e | %.2e | %.2e | %.2e | %d |" % (r["name"], r["act_err"], r["fro_rel"], r["max_rel"],
                                                                  r["median_rel"], r["saturated"]))
    return "\n".join(lines)


def main(argv=None) -> int:
    import workloads as wl
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--workload", default="dense_fprop", choices=["tiny_dense", "dense_fprop"])
    ap.add_argument("--rows-step", type=int, default=16, help="compare every n-th output row")
    args = ap.parse_args(argv)
    t0 = time.time()
    d = wl.CONFIGS[args.workload]()
    rows = np.arange(0, d.a.shape[0], args.rows_step, dtype=np.int64)
    res = study(d.a, d.b, rows)
    print("workload %s, %d sampled rows of %d, %.1f s" % (args.workload, rows.size, d.a.shape[0], time.time() - t0))
    print(table(res))
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
