"""Accumulation precision on B200 tensor cores (the drift demonstration).

"The Insider Secrets Of Deepseek Discovered" reports that FP8 GEMMs on H800
tensor cores keep only ~14 bits while accumulating, so error grows with the
inner dimension, and that promoting partial sums to FP32 at fixed K intervals
(Figure 7 (b)) removes it.  Here the same codes (per-tensor-quantized long-K
inputs, uniform[-1,1] + 0.5 so nothing cancels) go through

  * the promoted kernel (a fresh tensor-core accumulation every 128-deep slab,
    FP32 promotion in registers), and
  * the diagnostic kernel that accumulates all of K inside the tensor cores,

and both are compared with the oracle's exact product.  The promoted result
must meet the parity tolerance; the unpromoted error is measured and reported
(the pages give only an H800 figure, so it is not a pass/fail number).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import fp8_fine_grained_quant_b200 as fq
import workloads as wl
from parity import bf16_bits_of, gemm_errors, gemm_ok

pytestmark = pytest.mark.gpu
TILE = 128


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _u8(dev, a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def test_promotion_vs_tensor_core_accumulation(dev):
    d = wl.long_k(M=256, N=256, K=16384, seed=2)
    qa_full, s_a = oracle.quant_tensor(d.a)
    qb_full, s_b = oracle.quant_tensor(d.b)
    report = {}
    for K in (1024, 4096, 16384):
        qa = np.ascontiguousarray(qa_full[:, :K])
        qb = np.ascontiguousarray(qb_full[:, :K])
        sa = np.full((qa.shape[0], K // TILE), s_a, dtype=np.float32)
        sb = np.full((qb.shape[0] // TILE, K // TILE), s_b, dtype=np.float32)
        exact = oracle.gemm_blockscaled(qa, sa, qb, sb)
        args = [_u8(dev, qa), torch.from_numpy(sa).to(dev), _u8(dev, qb), torch.from_numpy(sb).to(dev)]
        promoted = fq.fp8_gemm_blockscaled(*args)
        unpromoted = fq.fp8_gemm_unpromoted_diag(*args)
        torch.cuda.synchronize(dev)
        assert fq.get_device_error(device=dev) == fq.OK
        p_bits, u_bits = bf16_bits_of(promoted), bf16_bits_of(unpromoted)
        st_p, st_u = gemm_errors(p_bits, exact), gemm_errors(u_bits, exact)
        assert gemm_ok(st_p), ("promoted", K, st_p)
        assert st_u["nonfinite"] == 0
        model = oracle.gemm_limited_acc(qa, sa, qb, sb, p_bits=14, group=32, interval=0, rows=np.arange(8))
        report[K] = {
            "promoted_implied_max_rel": st_p["implied_max_rel"],
            "promoted_not_correctly_rounded": st_p["not_correctly_rounded"],
            "unpromoted_implied_max_rel": st_u["implied_max_rel"],
            "unpromoted_out_max_rel": st_u["out_max_rel"],
            "unpromoted_not_correctly_rounded": st_u["not_correctly_rounded"],
            "oracle_14bit_model_max_rel": float(np.max(np.abs(model - exact[:8]) / np.abs(exact[:8]))),
        }
    print("accumulation report:", json.dumps(report))
    out = os.environ.get("FP8Q_RESULTS_DIR")
    if out:
        with open(os.path.join(out, "accumulation.json"), "w") as f:
            json.dump(report, f, indent=1)
