"""bench.py host logic on CPU: the reference (oracle) arm's JSON line, the
per-kernel algorithmic byte/FLOP accounting, and the multi-rank timing
reduction (max over ranks) on a world-size-2 gloo group."""
import json
import os
import subprocess
import sys
from pathlib import Path

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]
sys.path.insert(0, str(ROOT))
import bench  # noqa: E402
import workloads as wl  # noqa: E402


def test_reference_arm_prints_contract_line():
    out = subprocess.run([sys.executable, str(ROOT / "bench.py"), "--impl", "reference", "--workload", "tiny_dense",
                          "--steps", "3", "--warmup", "3"], capture_output=True, text=True, check=True, cwd=ROOT,
                         timeout=600)
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["config"]["workload"].startswith("tiny_dense")


def test_kernel_plan_accounting():
    d = wl.tiny_dense()
    M, N, K = 128, 256, 512
    act = M * K * 3 + M * (K // 128) * 4
    wt = N * K * 3 + (N // 128) * (K // 128) * 4
    try:
        bench._set_quant_mode("separate")
        plan = dict((k, (b, f)) for k, b, f in bench.kernel_plan("tiny_dense", d))
        assert plan["quant_act_1x128"][0] == act and plan["quant_w_128x128"][0] == wt
    finally:
        bench._set_quant_mode("fused")
    plan = dict((k, (b, f)) for k, b, f in bench.kernel_plan("tiny_dense", d))
    assert plan["quant_act_w"][0] == act + wt  # one launch for both operands
    assert plan["gemm_blockscaled"][1] == 2.0 * M * N * K
    assert plan["gemm_blockscaled"][0] == M * K + M * (K // 128) * 4 + N * K + (N // 128) * (K // 128) * 4 + M * N * 2


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        got = bench.max_over_ranks(float(10 * (rank + 1)), world, device="cpu")
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=5) for _ in range(2))
    assert res == {0: 20.0, 1: 20.0}


def test_cpu_sample_size_is_bounded():
    d = wl.tiny_dense()
    rows, nb = bench.cpu_sample_size("tiny_dense", d, 0.05)
    assert 1 <= rows <= d.M and 1 <= nb <= d.N // 128


def test_gemm_roofline_bound_follows_intensity():
    """Dense shapes are tensor-bound; the masked decode (few rows per expert)
    falls below the ridge and is reported against HBM."""
    from types import SimpleNamespace
    import numpy as np
    peaks = {"hbm_gbs": 6545.0, "source": "measured"}
    fp8 = 2 * 1627.8

    def kernels_for(plan, ms=1.0):
        return {l: {"avg_ms": ms, "tflops": (f / ms / 1e9) if f else 0.0, "gbs": b / ms / 1e6} for l, b, f in plan}

    dense = SimpleNamespace(M=4096, N=7168, K=7168)
    plan = bench.kernel_plan("dense_fprop", dense)
    r = bench.gemm_roofline(plan, kernels_for(plan), peaks, fp8, 1627.8, False, "dense_fprop")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["intensity_flop_per_byte"] > r["ridge_flop_per_byte"]

    E, cap, K, N, K2, N2 = 32, 256, 7168, 4096, 2048, 7168
    masked_m = np.full(E, 156, dtype=np.int32)
    shape = lambda *dims: SimpleNamespace(shape=dims)  # noqa: E731  (kernel_plan reads shapes only)
    masked = SimpleNamespace(a=shape(E, cap, K), b=shape(E, N, K), a2=shape(E, cap, K2), b2=shape(E, N2, K2),
                             masked_m=masked_m,
                             flops=lambda second: 2.0 * masked_m.sum() * (N2 * K2 if second else N * K))
    plan = bench.kernel_plan("moe_masked", masked)
    r = bench.gemm_roofline(plan, kernels_for(plan), peaks, fp8, 1627.8, False, "moe_masked")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and 0 < r["tensor_frac"] < 1
    assert r["intensity_flop_per_byte"] < r["ridge_flop_per_byte"]


def test_dgrad_plan_counts_the_transposed_gemm():
    from types import SimpleNamespace
    d = SimpleNamespace(M=4096, N=7168, K=7168)
    plan = bench.kernel_plan("dense_dgrad", d)
    labels = [l for l, _, _ in plan]
    assert labels == ["quant_act_w", "transpose_w_128x128", "gemm_dgrad"]
    assert plan[-1][2] == 2.0 * 4096 * 7168 * 7168
    assert plan[1][1] == 2 * 7168 * 7168 + 8 * 56 * 56


def test_traffic_is_reported_only_for_the_sources_it_was_taken_on(tmp_path, monkeypatch):
    """profiles/traffic.json entries carry the kernel sources' hash: an entry
    counts only while the sources hash to it (else the line's traffic is null)."""
    prof = tmp_path / "profiles"
    prof.mkdir()
    entry = {"dram_bytes_per_launch": 123, "source_hash": bench.source_hash()}
    (prof / "traffic.json").write_text(json.dumps({"gemm_blockscaled:dense_fprop": entry,
                                                  "quant_act_w:dense_fprop": dict(entry, source_hash="0" * 16)}))
    monkeypatch.setattr(bench, "ROOT", tmp_path)
    monkeypatch.setattr(bench, "source_hash", lambda: entry["source_hash"])
    assert bench.traffic_for("gemm_blockscaled", "dense_fprop") == 123
    assert bench.traffic_for("quant_act_w", "dense_fprop") is None      # taken on other sources
    assert bench.traffic_for("gemm_blockscaled", "long_k") is None       # never taken


def test_profile_sizes_shrink_the_workloads_they_name(monkeypatch):
    """--profile-size keeps each named workload's layout with fewer rows or
    experts (captures that take many passes stay small); the chained MoE decode
    takes the masked layout with 8 experts.  The generators are stubbed: only
    the arguments make_workload passes are checked."""
    calls = []
    monkeypatch.setattr(wl, "moe_masked", lambda **kw: calls.append(("moe_masked", kw)) or "masked")
    monkeypatch.setitem(wl.CONFIGS, "dense_fprop", lambda **kw: calls.append(("dense_fprop", kw)) or "dense")
    monkeypatch.setattr(bench, "PROFILE_SIZE", True)
    assert bench.make_workload("moe_masked_chain") == "masked"
    assert bench.make_workload("dense_fprop") == "dense"
    assert calls == [("moe_masked", {"device": None, "E": 8}), ("dense_fprop", {"M": 2048})]
    monkeypatch.setattr(bench, "PROFILE_SIZE", False)
    calls.clear()
    assert bench.make_workload("moe_masked_chain") == "masked"
    assert calls == [("moe_masked", {"shard": 0, "device": None})]
