#!/usr/bin/env python
"""Benchmark of the fine-grained FP8 path on B200: one step = online 1x128
activation quantization + online 128x128 weight quantization + block-scaled
FP8 GEMM with per-slab promotion, on one batch of synthetic input.

Default workload: dense Fprop M=4096 (tokens), K=7168, N=7168 (the dense
configuration the headline metric is quoted on).  ``--workload`` selects the
others (tiny_dense, long_k, moe_contiguous, moe_masked) for extra lines.

Prints ONE JSON line (rank 0).  Timing: W untimed warm-up steps, then K timed
steps bracketed by barrier + device synchronize, CUDA events on the launching
stream, max over ranks.  Inputs rotate over enough buffer sets that a step's
inputs were not touched by the step before (the per-set footprint exceeds the
126 MB L2).

Multi-GPU: launched by torchrun, every rank runs its own independent problem
of the same size (weak scaling; the path has no exchange step, so no
collective touches the data).

``--impl reference`` times the CPU oracle (the only reference implementation
this path has) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

TILE = 128
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FP8_OVER_BF16 = 2.0  # nominal dense fp8 / bf16 tensor throughput ratio (4.5 / 2.25 PFLOP/s)
SUSTAINED_AFTER_S = 1.0


# ---------------------------------------------------------------------------- helpers
METRIC = "FP8 block-scaled GEMM TFLOPS (step = 1x128 act quant + 128x128 weight quant + GEMM)"


def load_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return {"hbm_gbs": d["hbm_gbs"], "bf16": d["bf16_tflops"],
                "bf16_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16": FALLBACK_BF16_TFLOPS, "bf16_sustained": 1400.0,
            "source": "fallback"}


def source_hash() -> str:
    h = hashlib.sha256()
    for p in sorted((ROOT / "fp8_fine_grained_quant_b200" / "csrc").glob("*")) + [ROOT / "include" / "fp8q.h"]:
        h.update(p.read_bytes())
    return h.hexdigest()[:16]


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


class ClockSampler:
    """Samples SM clock and clock-event (throttle) reasons through NVML while
    the timed region runs (reading only; nothing is changed)."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.002):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self._stop = threading.Event()
        self.max_mhz = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = repr(e)

    def _sample(self):
        nv = self._nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        except Exception:  # noqa: BLE001
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
        for bit, name in self.REASONS.items():
            if r & bit:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._sample()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()
            self._sample()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "note": getattr(self, "err", "")}
        busy = sorted(self.reasons - {"gpu_idle"})
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz, "reasons": busy,
                "samples": len(self.samples), "sm_mhz_min": min(self.samples)}


# ---------------------------------------------------------------------------- workloads
# Reduced sizes of the same workloads for ncu captures that take many passes
# (a few GB on the device at most); never a bench line of their own.
PROFILE_SIZES = {
    "dense_fprop": dict(M=2048), "long_k": dict(M=1024), "moe_contiguous": dict(tokens=1024, E=8),
    "moe_masked": dict(E=8), "moe_masked_chain": dict(E=8),
}
PROFILE_SIZE = False


def make_workload(name: str, shard: int = 0, device=None):
    """The named workload; ``shard`` r > 0 is rank r's part of the batch
    (row blocks for the dense shapes, experts for the MoE ones; see
    workloads.row_shard / expert_shard).  ``device`` draws the large MoE
    tensors on that device instead of the host."""
    import workloads as wl
    if PROFILE_SIZE and name in PROFILE_SIZES:
        kw = PROFILE_SIZES[name]
        if name == "moe_masked_chain":
            return wl.moe_masked(device=device, **kw)
        if name.startswith("moe"):
            return wl.CONFIGS[name](device=device, **kw)
        return wl.CONFIGS[name](**kw)
    if name in ("dense_fprop", "dense_dgrad", "dense_fprop_mx"):
        # dense_dgrad: the activation-gradient GEMM of the dense_fprop layer;
        # dY takes the shape and distribution of the forward activations.
        # dense_fprop_mx: the same GEMM with power-of-two scales applied by
        # the tensor cores
        return wl.dense_fprop(shard=shard)
    if name == "long_k":
        return wl.long_k(shard=shard)
    if name == "dense_wgrad":
        return wl.dense_wgrad(seed=5 + 100 * shard) if shard else wl.dense_wgrad()
    if name in ("moe_masked", "moe_masked_chain"):
        # moe_masked_chain: GEMM2's activation is the SwiGLU of GEMM1's output,
        # requantized (its own A2 draw is not used)
        return wl.moe_masked(shard=shard, device=device)
    if name in ("moe_contiguous", "moe_contiguous_mx"):
        return wl.moe_contiguous(shard=shard, device=device)
    return wl.CONFIGS[name]()


def describe(name: str, d) -> dict:
    if name in ("tiny_dense", "dense_fprop", "long_k", "dense_fprop_mx"):
        return {"workload": "%s M=%d N=%d K=%d" % (name, d.M, d.N, d.K), "M": d.M, "N": d.N, "K": d.K,
                "seed": d.meta["seed"]}
    if name == "dense_dgrad":
        return {"workload": "dense_dgrad dX[M,K] = dY[M,N] W[N,K] M=%d N=%d K=%d" % (d.M, d.N, d.K), "M": d.M,
                "N": d.N, "K": d.K, "seed": d.meta["seed"]}
    if name == "dense_wgrad":
        return {"workload": "dense_wgrad dW[N,K] = dY[M,N]^T X[M,K] M=%d N=%d K=%d" % (d.M, d.N, d.K), "M": d.M,
                "N": d.N, "K": d.K, "seed": d.meta["seed"]}
    if name in ("moe_contiguous", "moe_contiguous_mx"):
        return {"workload": "%s E=%d M_tot=%d (valid %d) N=%d K=%d" % (name, d.E, d.M_tot, int(d.counts.sum()),
                                                                     d.N, d.K),
                "E": d.E, "M_tot": d.M_tot, "valid_rows": int(d.counts.sum()), "N": d.N, "K": d.K,
                "seed": d.meta["seed"]}
    return {"workload": "%s E=%d cap=%d valid=%d (N,K)=(%d,%d)+(%d,%d)" % (
        name, d.E, d.cap, int(d.masked_m.sum()), d.b.shape[1], d.b.shape[2], d.b2.shape[1], d.b2.shape[2]),
        "E": d.E, "cap": d.cap, "valid_rows": int(d.masked_m.sum()), "seed": d.meta["seed"]}


def _to_dev_bf16(torch, bits, dev):
    """bf16 bit patterns (numpy) or a bf16 tensor already drawn on the device
    (a copy, so rotating input sets are distinct buffers)."""
    if isinstance(bits, torch.Tensor):
        return bits.to(dev).clone()
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)


def _to_dev_i32(torch, arr, dev):
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.int32)).to(dev)


def build_sets(name, d, dev, nsets, torch, fq):
    """Per input set: device tensors and preallocated outputs."""
    sets = []
    for _ in range(nsets):
        s = {}
        if name in ("moe_masked", "moe_masked_chain"):
            E, cap, K = d.a.shape
            s["a"] = _to_dev_bf16(torch, d.a.reshape(E * cap, K), dev)
            s["b"] = _to_dev_bf16(torch, d.b, dev)
            if name == "moe_masked":
                s["a2"] = _to_dev_bf16(torch, d.a2.reshape(E * cap, -1), dev)
            s["b2"] = _to_dev_bf16(torch, d.b2, dev)
            s["mm"] = _to_dev_i32(torch, d.masked_m, dev)
        elif name == "dense_wgrad":
            s["dy"] = _to_dev_bf16(torch, d.dy, dev)
            s["x"] = _to_dev_bf16(torch, d.x, dev)
        else:
            s["a"] = _to_dev_bf16(torch, d.a, dev)
            s["b"] = _to_dev_bf16(torch, d.b, dev)
            if name in ("moe_contiguous", "moe_contiguous_mx"):
                s["mi"] = _to_dev_i32(torch, d.m_indices, dev)
        sets.append(s)
    return sets


# How a step quantizes a GEMM's two operands: "fused" = one launch of
# fp8_quant_act_w for both, "separate" = fp8_quant_act_1x128 then
# fp8_quant_w_128x128.  Set from --quant.
QUANT_MODE = "fused"


def kernel_plan(name, d):
    """(kernel label, algorithmic bytes, algorithmic FLOPs) per launch of one step."""
    def qa_bytes(rows, K):
        return rows * K * (2 + 1) + rows * (K // TILE) * 4

    def qw_bytes(G, N, K):
        return G * N * K * (2 + 1) + G * (N // TILE) * (K // TILE) * 4

    def gemm_bytes(rows, N, K, G=1):
        return rows * K + rows * (K // TILE) * 4 + G * N * K + G * (N // TILE) * (K // TILE) * 4 + rows * N * 2

    def quant(a_bytes, w_bytes, suffix=""):
        if QUANT_MODE == "fused":
            return [("quant_act_w" + suffix, a_bytes + w_bytes, 0.0)]
        return [("quant_act_1x128" + suffix, a_bytes, 0.0), ("quant_w_128x128" + suffix, w_bytes, 0.0)]

    if name in ("tiny_dense", "dense_fprop", "long_k"):
        M, N, K = d.M, d.N, d.K
        return quant(qa_bytes(M, K), qw_bytes(1, N, K)) + [("gemm_blockscaled", gemm_bytes(M, N, K), 2.0 * M * N * K)]
    if name in ("dense_fprop_mx", "moe_contiguous_mx"):
        # power-of-two scales: the _ue8m0 quantizers, the scales' E8M0 atoms,
        # then the GEMM with the scales applied in the tensor cores
        contiguous = name == "moe_contiguous_mx"
        rows, G = (d.M_tot, d.E) if contiguous else (d.M, 1)
        N, K = d.N, d.K
        nkb = K // TILE
        atoms_a, atoms_b = -(-rows // TILE) * nkb * 512, G * (N // TILE) * nkb * 512
        gemm = rows * K + G * N * K + atoms_a + atoms_b + rows * N * 2
        return [("quant_act_1x128_ue8m0", qa_bytes(rows, K), 0.0), ("quant_w_128x128_ue8m0", qw_bytes(G, N, K), 0.0),
                ("mx_scales_act", rows * nkb * 4 + atoms_a, 0.0),
                ("mx_scales_w", G * (N // TILE) * nkb * 4 + atoms_b, 0.0),
                ("grouped_gemm_mx_contiguous" if contiguous else "gemm_mx", gemm,
                 d.flops if contiguous else 2.0 * rows * N * K)]
    if name == "dense_dgrad":
        # dY is d.a [M, Nout], W is d.b [Nout, K]; dX = dY W is [M, K]
        M, Nout, K = d.M, d.N, d.K
        return quant(qa_bytes(M, Nout), qw_bytes(1, Nout, K)) + [
            ("transpose_w_128x128", 2 * Nout * K + 2 * 4 * (Nout // TILE) * (K // TILE), 0.0),
            ("gemm_dgrad", gemm_bytes(M, K, Nout), 2.0 * M * Nout * K)]
    if name == "dense_wgrad":
        # both operands quantized along tokens, codes written token-contiguous
        M, N, K = d.M, d.N, d.K
        Mp = -(-M // (4 * TILE)) * (4 * TILE)  # tokens in whole groups of four slabs

        def qt_bytes(C):
            return M * C * 2 + C * Mp + (Mp // TILE) * C * 4

        gemm = N * Mp + K * Mp + (Mp // TILE) * (N + K) * 4 + N * K * 2
        return [("quant_act_128x1_t", qt_bytes(N), 0.0), ("quant_act_128x1_t#2", qt_bytes(K), 0.0),
                ("gemm_wgrad", gemm, 2.0 * M * N * K)]
    if name == "moe_contiguous":
        return quant(qa_bytes(d.M_tot, d.K), qw_bytes(d.E, d.N, d.K)) + [
            ("grouped_gemm_contiguous", gemm_bytes(d.M_tot, d.N, d.K, d.E), d.flops)]
    E, cap, K = d.a.shape
    N, K2, N2 = d.b.shape[1], d.a2.shape[2], d.b2.shape[1]
    active = int((d.masked_m > 0).sum())
    valid = int(d.masked_m.sum())
    if name == "moe_masked_chain":
        # GEMM1's valid rows in (gate | up, bf16), h's codes and scales out
        swiglu = valid * N * 2 + valid * K2 + valid * (K2 // TILE) * 4
        return quant(qa_bytes(E * cap, K), qw_bytes(E, N, K)) + [
            ("grouped_gemm_masked", gemm_bytes(valid, N, K, active), d.flops(False)),
            ("swiglu_quant_1x128", swiglu, 0.0), ("quant_w_128x128#2", qw_bytes(E, N2, K2), 0.0),
            ("grouped_gemm_masked#2", gemm_bytes(valid, N2, K2, active), d.flops(True))]
    return (quant(qa_bytes(E * cap, K), qw_bytes(E, N, K)) +
            [("grouped_gemm_masked", gemm_bytes(valid, N, K, active), d.flops(False))] +
            quant(qa_bytes(E * cap, K2), qw_bytes(E, N2, K2), "#2") +
            [("grouped_gemm_masked#2", gemm_bytes(valid, N2, K2, active), d.flops(True))])


def launch_step(name, d, s, fq, events=None):
    """Launch the kernels of one step on the current stream.  `events`, if
    given, is a list of (start, end) CUDA-event pairs, one per kernel, in
    kernel_plan's order."""
    k = [0]

    def rec(which):
        if events is not None:
            events[k[0]][which].record()
        if which:
            k[0] += 1

    def quant(a, b, qa, sa, qb, sb):
        """Both operands of a GEMM; returns (qa, sa, qb, sb)."""
        if QUANT_MODE == "fused":
            rec(0)
            (q1, s1), (q2, s2) = fq.fp8_quant_act_w(s[a], s[b], s.get(qa), s.get(sa), s.get(qb), s.get(sb))
            rec(1)
        else:
            rec(0); q1, s1 = fq.fp8_quant_act_1x128(s[a], s.get(qa), s.get(sa)); rec(1)
            rec(0); q2, s2 = fq.fp8_quant_w_128x128(s[b], s.get(qb), s.get(sb)); rec(1)
        s.update({qa: q1, sa: s1, qb: q2, sb: s2})
        return q1, s1, q2, s2

    if name == "moe_masked_chain":
        E, cap, K = d.a.shape
        qa, sa, qb, sb = quant("a", "b", "qa", "sa", "qb", "sb")
        rec(0)
        c = fq.fp8_grouped_gemm_masked(qa.view(E, cap, K), sa.view(E, cap, K // TILE), qb, sb, s["mm"],
                                       expected_m=int(d.masked_m.mean()), out=s.get("c"))
        rec(1)
        rec(0); qh, sh = fq.fp8_swiglu_quant_1x128(c, s["mm"], s.get("qh"), s.get("sh")); rec(1)
        rec(0); qb2, sb2 = fq.fp8_quant_w_128x128(s["b2"], s.get("qb2"), s.get("sb2")); rec(1)
        rec(0)
        c2 = fq.fp8_grouped_gemm_masked(qh, sh, qb2, sb2, s["mm"], expected_m=int(d.masked_m.mean()),
                                        out=s.get("c2"))
        rec(1)
        s.update(c=c, qh=qh, sh=sh, qb2=qb2, sb2=sb2, c2=c2)
        return c2
    if name == "moe_masked":
        E, cap, K = d.a.shape
        qa, sa, qb, sb = quant("a", "b", "qa", "sa", "qb", "sb")
        rec(0)
        c = fq.fp8_grouped_gemm_masked(qa.view(E, cap, K), sa.view(E, cap, K // TILE), qb, sb, s["mm"],
                                       expected_m=int(d.masked_m.mean()), out=s.get("c"))
        rec(1)
        K2 = d.a2.shape[2]
        qa2, sa2, qb2, sb2 = quant("a2", "b2", "qa2", "sa2", "qb2", "sb2")
        rec(0)
        c2 = fq.fp8_grouped_gemm_masked(qa2.view(E, cap, K2), sa2.view(E, cap, K2 // TILE), qb2, sb2, s["mm"],
                                        expected_m=int(d.masked_m.mean()), out=s.get("c2"))
        rec(1)
        s.update(c=c, c2=c2)
        return c2
    if name in ("dense_fprop_mx", "moe_contiguous_mx"):
        rec(0); qa, sa = fq.fp8_quant_act_1x128_ue8m0(s["a"], s.get("qa"), s.get("sa")); rec(1)
        rec(0); qb, sb = fq.fp8_quant_w_128x128_ue8m0(s["b"], s.get("qb"), s.get("sb")); rec(1)
        rec(0); sfa = fq.fp8_mx_scales_act(sa, s.get("sfa")); rec(1)
        rec(0); sfb = fq.fp8_mx_scales_w(sb, s.get("sfb")); rec(1)
        rec(0)
        if name == "moe_contiguous_mx":
            c = fq.fp8_grouped_gemm_mx_contiguous(qa, sfa, qb, sfb, s["mi"], out=s.get("c"))
        else:
            c = fq.fp8_gemm_mx(qa, sfa, qb, sfb, out=s.get("c"))
        rec(1)
        s.update(qa=qa, sa=sa, qb=qb, sb=sb, sfa=sfa, sfb=sfb, c=c)
        return c
    if name == "dense_wgrad":
        rec(0); q_dy, s_dy = fq.fp8_quant_act_128x1_t(s["dy"], s.get("q_dy"), s.get("s_dy")); rec(1)
        rec(0); q_x, s_x = fq.fp8_quant_act_128x1_t(s["x"], s.get("q_x"), s.get("s_x")); rec(1)
        rec(0); c = fq.fp8_gemm_wgrad(q_dy, s_dy, q_x, s_x, out=s.get("c")); rec(1)
        s.update(q_dy=q_dy, s_dy=s_dy, q_x=q_x, s_x=s_x, c=c)
        return c
    qa, sa, qb, sb = quant("a", "b", "qa", "sa", "qb", "sb")
    if name == "dense_dgrad":
        rec(0); qt, st = fq.fp8_transpose_w_128x128(qb, sb, s.get("qt"), s.get("st")); rec(1)
        rec(0); c = fq.fp8_gemm_blockscaled(qa, sa, qt, st, out=s.get("c")); rec(1)
        s.update(qt=qt, st=st, c=c)
        return c
    rec(0)
    if name == "moe_contiguous":
        c = fq.fp8_grouped_gemm_contiguous(qa, sa, qb, sb, s["mi"], out=s.get("c"))
    else:
        c = fq.fp8_gemm_blockscaled(qa, sa, qb, sb, out=s.get("c"))
    rec(1)
    s.update(c=c)
    return c


def step_flops(name, d):
    if name in ("moe_masked", "moe_masked_chain"):
        return d.flops(False) + d.flops(True)
    return d.flops


# ---------------------------------------------------------------------------- CPU oracle timing
def oracle_sample_step(name, d, rows: int, nblocks: int):
    """One oracle step on a bounded sample of the workload: the activation
    quantization of `rows` rows, the weight quantization of `nblocks` 128-row
    weight blocks, and the GEMM outputs rows x (128 * nblocks).  Returns
    (seconds, flops of the sample)."""
    import oracle
    if name == "dense_wgrad":
        # `rows` output channels of dY and `nblocks` x 128 of X, over every token
        dy = np.ascontiguousarray(d.dy[:, :rows])
        x = np.ascontiguousarray(d.x[:, :TILE * nblocks])
        t0 = time.perf_counter()
        q_dy, s_dy = oracle.quant_act_128x1(dy)
        q_x, s_x = oracle.quant_act_128x1(x)
        oracle.wgrad(q_dy, s_dy, q_x, s_x)
        dt = time.perf_counter() - t0
        return dt, 2.0 * rows * TILE * nblocks * d.M
    if name in ("moe_masked", "moe_masked_chain"):
        a, b = d.a[0], d.b[0]
    elif name in ("moe_contiguous", "moe_contiguous_mx"):
        a, b = d.a, d.b[int(d.m_indices[0])]
    else:
        a, b = d.a, d.b
    K = a.shape[1]
    ra = np.ascontiguousarray(a[:rows])
    rb = np.ascontiguousarray(b[:TILE * nblocks])
    t0 = time.perf_counter()
    qa, sa = oracle.quant_act_1x128(ra)
    qb, sb = oracle.quant_w_128x128(rb)
    oracle.gemm_blockscaled(qa, sa, qb, sb)
    dt = time.perf_counter() - t0
    return dt, 2.0 * rows * TILE * nblocks * K


def sample_description(name, d, rows: int, nb: int) -> str:
    if name == "dense_wgrad":
        return ("token-axis quantization of %d dY channels and %d X channels over %d tokens, float64 weight-"
                "gradient GEMM of the %d x %d outputs they determine" % (rows, TILE * nb, d.M, rows, TILE * nb))
    return ("1x128 quantization of %d rows of A, 128x128 quantization of %d weight block-rows (%d x %d), "
            "float64 GEMM of the %d x %d outputs they determine (K=%d)" % (
                rows, nb, TILE * nb, d.a.shape[-1], rows, TILE * nb, d.a.shape[-1]))


def cpu_sample_size(name, d, budget_s: float):
    """Rows x weight blocks whose oracle step takes about budget_s."""
    rows, nb = 8, 1
    if name == "dense_wgrad":
        nb_max, rows_max = d.K // TILE, d.N
    else:
        nb_max = (d.b.shape[-2]) // TILE
        rows_max = d.a.shape[-2]
    # a step's cost is not proportional to rows x blocks at small sizes
    # (fixed costs dominate), so grow the sample in a few measured rounds
    for _ in range(5):
        dt, _ = oracle_sample_step(name, d, rows, nb)
        if dt >= 0.7 * budget_s or (rows == rows_max and nb == nb_max):
            break
        scale = min(16.0, budget_s / max(dt, 1e-4))
        new_nb = int(min(nb_max, max(nb, round(nb * scale ** 0.5))))
        rows = int(min(rows_max, max(1, round(rows * scale * nb / new_nb))))
        nb = new_nb
    return rows, nb


def run_reference(args, name):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    d = make_workload(name)
    per_step = max(0.05, min(2.0, 120.0 / max(1, args.steps + args.warmup)))
    rows, nb = cpu_sample_size(name, d, per_step)
    for _ in range(args.warmup):
        oracle_sample_step(name, d, rows, nb)
    times, flops = [], 0.0
    for _ in range(args.steps):
        dt, f = oracle_sample_step(name, d, rows, nb)
        times.append(dt)
        flops += f
    total = sum(times)
    value = flops / total / 1e12
    sample = "per step: " + sample_description(name, d, rows, nb)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(describe(name, d), parallelism="single"),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ---------------------------------------------------------------------------- GPU arm
def traffic_for(kernel: str, name: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources; otherwise None."""
    p = ROOT / "profiles" / "traffic.json"
    if not p.exists():
        return None
    try:
        t = json.loads(p.read_text())
        ent = t.get("%s:%s" % (kernel, name))
        if ent and ent.get("source_hash") == source_hash():
            return ent["dram_bytes_per_launch"]
    except Exception:  # noqa: BLE001
        return None
    return None


def gemm_roofline(plan, kernels, peaks, fp8_peak, bf16_peak, sustained, name):
    """Roofline entry for the step's GEMM (the dominant kernel).  Its bound
    follows from its arithmetic intensity against the ridge of the two
    measured peaks: tensor-bound for the dense and contiguous shapes,
    HBM-bound for the masked decode (few rows per expert, every active
    expert's weights read once)."""
    gemm_label, gemm_bytes, gemm_flops = [(l, b, f) for l, b, f in plan if f][0]
    g = kernels[gemm_label]
    intensity = gemm_flops / gemm_bytes
    ridge = fp8_peak * 1e12 / (peaks["hbm_gbs"] * 1e9)
    peak_note = "%s (%s bf16 %.1f TFLOP/s x %.0f fp8/bf16 nominal ratio)" % (
        peaks["source"], "sustained" if sustained else "burst", bf16_peak, FP8_OVER_BF16)
    if intensity >= ridge:
        roofline = {"bound": "tensor", "kernel": gemm_label, "achieved": g["tflops"], "peak": fp8_peak,
                    "unit": "TFLOP/s", "frac": g["tflops"] / fp8_peak, "peak_source": peak_note}
    else:
        roofline = {"bound": "hbm", "kernel": gemm_label, "achieved": g["gbs"], "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": g["gbs"] / peaks["hbm_gbs"],
                    "peak_source": "%s copy bandwidth" % peaks["source"],
                    "tensor_frac": g["tflops"] / fp8_peak, "tensor_peak_source": peak_note}
    roofline.update(traffic=traffic_for(gemm_label, name), algorithmic_flops_per_launch=gemm_flops,
                    algorithmic_bytes_per_launch=gemm_bytes, intensity_flop_per_byte=intensity,
                    ridge_flop_per_byte=ridge)
    return roofline


def enqueue_ahead(torch, ms: float = 20.0):
    """A short device-side delay before the timed region, so the host has the
    first steps' launches queued when the device reaches them: the events
    then time the kernels, not the host's launch latency.  The delay itself
    lies before the start event."""
    torch.cuda._sleep(int(ms * 1e6))  # ~1 cycle per ns at the SM clock: a delay of a few ms to tens of ms


def measure(name, d, dev, steps, warmup, world, torch, fq):
    """Times `steps` steps of the workload (after `warmup` untimed ones) on
    rotating input sets: the step's elapsed device time (max over ranks),
    every kernel's per-launch times, the clock record and the launch count."""
    plan = kernel_plan(name, d)
    nk = len(plan)
    per_set_bytes = sum(b for _, b, _ in plan)
    nsets = max(2, int(np.ceil(2 * 126e6 / max(per_set_bytes, 1))))
    nsets = min(nsets, 4)
    sets = build_sets(name, d, dev, nsets, torch, fq)
    stream = torch.cuda.current_stream(dev)

    for i in range(warmup):
        launch_step(name, d, sets[i % nsets], fq)
    torch.cuda.synchronize(dev)
    if fq.get_device_error(device=dev) != fq.OK:
        raise RuntimeError("device error during warm-up of %s" % name)

    events = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)] for _ in range(nk)]
              for _ in range(steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    launches0 = fq.launch_count()
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clk:
        enqueue_ahead(torch)
        t_start.record(stream)
        for i in range(steps):
            launch_step(name, d, sets[i % nsets], fq, events[i])
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    launches = fq.launch_count() - launches0
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end), world, dev)
    if fq.get_device_error(device=dev) != fq.OK:
        raise RuntimeError("device error in the timed region of %s" % name)
    kernel_ms = [[events[i][k][0].elapsed_time(events[i][k][1]) for i in range(steps)] for k in range(nk)]
    # per kernel: the max over ranks of its mean launch time
    kernel_ms = [[max_over_ranks(float(np.mean(ms)), world, dev)] for ms in kernel_ms]
    del sets
    return {"plan": plan, "elapsed_ms": elapsed_ms, "kernel_ms": kernel_ms, "clocks": clk.summary(),
            "launches": int(launches), "nsets": nsets, "per_set_bytes": per_set_bytes}


def kernel_table(m, peaks, fp8_peak):
    kernels = {}
    for k, (label, nbytes, kflops) in enumerate(m["plan"]):
        avg_ms = float(np.mean(m["kernel_ms"][k]))
        ent = {"avg_ms": avg_ms, "bytes": nbytes}
        if kflops:
            ent.update(tflops=kflops / avg_ms / 1e9, frac_of_fp8_peak=kflops / avg_ms / 1e9 / fp8_peak)
        ent.update(gbs=nbytes / avg_ms / 1e6, frac_of_hbm=nbytes / avg_ms / 1e6 / peaks["hbm_gbs"])
        kernels[label] = ent
    return kernels


def peaks_for(elapsed_ms):
    """Peaks for a timed region: the burst bf16 figure for a short region,
    the sustained one for a region of a second or more."""
    peaks = load_peaks()
    sustained = elapsed_ms / 1e3 >= SUSTAINED_AFTER_S
    bf16_peak = peaks["bf16_sustained"] if sustained else peaks["bf16"]
    return peaks, bf16_peak * FP8_OVER_BF16, bf16_peak, sustained


def _set_quant_mode(mode):
    global QUANT_MODE
    QUANT_MODE = mode


# Secondary workloads the default run times after the headline (their own
# per-kernel tables, rooflines and clocks under one key of the same line).
SECONDARY = ("long_k", "moe_contiguous", "moe_masked")
SECONDARY_STEPS, SECONDARY_WARMUP = 10, 3


def secondary_lines(args, dev, world, rank, torch, fq):
    out = {}
    for name in SECONDARY:
        d = make_workload(name, shard=rank, device=dev if name.startswith("moe") else None)
        m = measure(name, d, dev, SECONDARY_STEPS, SECONDARY_WARMUP, world, torch, fq)
        peaks, fp8_peak, bf16_peak, sustained = peaks_for(m["elapsed_ms"])
        kernels = kernel_table(m, peaks, fp8_peak)
        flops = step_flops(name, d)
        draws = d.meta.get("draws", "host")
        out[name] = {
            "value": world * flops * SECONDARY_STEPS / (m["elapsed_ms"] / 1e3) / 1e12, "unit": "TFLOP/s",
            "ms_per_step": m["elapsed_ms"] / SECONDARY_STEPS, "steps": SECONDARY_STEPS, "warmup": SECONDARY_WARMUP,
            "config": dict(describe(name, d), draws=draws,
                           l2="inputs rotated over %d buffer sets (%.0f MB each) between steps" % (
                               m["nsets"], m["per_set_bytes"] / 1e6)),
            "roofline": gemm_roofline(m["plan"], kernels, peaks, fp8_peak, bf16_peak, sustained, name),
            "kernels": kernels, "gpu_launches": m["launches"], "clocks": m["clocks"],
        }
        del d
        torch.cuda.empty_cache()
    return out


def run_ours(args, name):
    import torch
    rank, world, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    import fp8_fine_grained_quant_b200 as fq
    fq.lib()

    # rank r runs its shard of a batch `world` times the single-GPU one: row
    # blocks (dense; B replicated) or experts (MoE); no collective touches
    # the data, only the barrier and the max-over-ranks of the timings
    d = make_workload(name, shard=rank)
    m = measure(name, d, dev, args.steps, args.warmup, world, torch, fq)
    flops = step_flops(name, d)

    # the same step with the operands quantized by the two separate kernels
    # (their own launch times, for comparison with the one-launch quantizer)
    other = None
    if QUANT_MODE == "fused" and name in ("dense_fprop", "long_k", "moe_contiguous", "moe_masked", "dense_dgrad"):
        try:
            _set_quant_mode("separate")
            other = measure(name, d, dev, args.steps, args.warmup, world, torch, fq)
        finally:
            _set_quant_mode("fused")

    # ------------------------------------------------------------ e2e (host buffers)
    e2e = run_e2e(args, name, d, dev, torch, fq, world)
    extra = None
    if name == "dense_fprop" and not args.no_secondary:
        extra = secondary_lines(args, dev, world, rank, torch, fq)

    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return 0

    peaks, fp8_peak, bf16_peak, sustained = peaks_for(m["elapsed_ms"])
    kernels = kernel_table(m, peaks, fp8_peak)
    roofline = gemm_roofline(m["plan"], kernels, peaks, fp8_peak, bf16_peak, sustained, name)
    value = world * flops * args.steps / (m["elapsed_ms"] / 1e3) / 1e12
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(name, d)
    line = {
        "metric": METRIC,
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": m["elapsed_ms"] / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
        "config": dict(describe(name, d),
                       parallelism=("dp%d: %s shard per rank, no data-path collective" % (
                           world, "expert" if name.startswith("moe") else "M-row")) if world > 1 else "single",
                       l2="inputs rotated over %d buffer sets (%.0f MB each) between steps" % (
                           m["nsets"], m["per_set_bytes"] / 1e6)),
        "roofline": roofline, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": m["launches"], "clocks": m["clocks"],
    }
    if other is not None:
        op, ofp8, obf16, osus = peaks_for(other["elapsed_ms"])
        line["separate_quantizers"] = {
            "note": "the same step with fp8_quant_act_1x128 and fp8_quant_w_128x128 launched separately",
            "value": world * flops * args.steps / (other["elapsed_ms"] / 1e3) / 1e12, "unit": "TFLOP/s",
            "ms_per_step": other["elapsed_ms"] / args.steps, "kernels": kernel_table(other, op, ofp8),
            "clocks": other["clocks"]}
    if extra is not None:
        line["secondary_workloads"] = extra
    if PROFILE_SIZE:
        line["profile_size"] = "reduced shapes for a profiler capture: not a bench line"
    print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_e2e(args, name, d, dev, torch, fq, world):
    """Same step through the public API from pinned host buffers: H2D copy of
    the bf16 inputs, the three kernels, D2H copy of the bf16 result."""
    host = {}
    if name == "dense_wgrad":
        keys, src = ["dy", "x"], {"dy": d.dy, "x": d.x}
    else:
        keys = ["a", "b"] + (["a2", "b2"] if name == "moe_masked" else ["b2"] if name == "moe_masked_chain" else [])
        src = {"a": d.a, "b": d.b}
        if name in ("moe_masked", "moe_masked_chain"):
            src.update(a2=d.a2, b2=d.b2)
    for k in keys:
        arr = np.ascontiguousarray(src[k]).view(np.int16)
        host[k] = torch.from_numpy(arr).pin_memory()
    s = build_sets(name, d, dev, 1, torch, fq)[0]
    out_host = None
    h2d = sum(host[k].numel() * 2 for k in keys)
    steps = max(3, min(args.steps, 20))

    def one():
        nonlocal out_host
        for k in keys:
            s[k].view(torch.int16).view(host[k].shape).copy_(host[k], non_blocking=True)
        c = launch_step(name, d, s, fq)
        if out_host is None:
            out_host = torch.empty(c.shape, dtype=c.dtype).pin_memory()
        out_host.copy_(c, non_blocking=True)

    for _ in range(2):
        one()
    torch.cuda.synchronize(dev)
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        one()
    e1.record()
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / steps
    value = world * step_flops(name, d) / (ms / 1e3) / 1e12
    return {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(out_host.numel() * 2), "ms_per_step": ms, "steps": steps}


def cpu_baseline(name, d):
    import oracle
    budget = float(os.environ.get("FP8Q_CPU_BASELINE_S", "15"))
    rows, nb = cpu_sample_size(name, d, budget / 3)
    dts, fl = [], 0.0
    for _ in range(3):
        dt, f = oracle_sample_step(name, d, rows, nb)
        dts.append(dt)
        fl += f
    value = fl / sum(dts) / 1e12
    return {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "3 oracle steps, each: %s; %.1f s total" % (sample_description(name, d, rows, nb), sum(dts))}


def relaunch_under_torchrun(args_list, n: int) -> int:
    """`bench.py --gpus N` outside a launcher: start N ranks on this node
    with torch.distributed.run (rendezvous on 127.0.0.1) and return its
    status; rank 0 prints the line."""
    import socket
    import subprocess
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(n),
           "--master-addr", "127.0.0.1", "--master-port", str(port), str(Path(__file__).resolve())] + list(args_list)
    return subprocess.call(cmd)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="dense_fprop",
                    choices=["tiny_dense", "dense_fprop", "long_k", "moe_contiguous", "moe_masked", "dense_dgrad",
                             "moe_masked_chain", "dense_wgrad", "dense_fprop_mx", "moe_contiguous_mx"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--quant", choices=["fused", "separate"], default="fused",
                    help="quantize a GEMM's two operands in one launch (fp8_quant_act_w) or in two")
    ap.add_argument("--profile-size", action="store_true",
                    help="reduced shapes of the same workload, for ncu captures (the line says so)")
    ap.add_argument("--no-secondary", action="store_true",
                    help="time the named workload only (the default dense_fprop run also times long_k, "
                         "moe_contiguous and moe_masked)")
    raw = sys.argv[1:] if argv is None else list(argv)
    args = ap.parse_args(raw)
    if args.warmup < 3:
        args.warmup = 3
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return relaunch_under_torchrun(raw, args.gpus)
    global QUANT_MODE, PROFILE_SIZE
    QUANT_MODE = args.quant
    PROFILE_SIZE = args.profile_size
    if args.impl == "reference":
        return run_reference(args, args.workload)
    return run_ours(args, args.workload)


if __name__ == "__main__":
    sys.exit(main())
