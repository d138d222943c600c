"""The multi-GPU partition of the path on CPU: the dense batch is split into
M-row blocks (whole 128-row tiles, B replicated) and the MoE layers into
expert ranges, one per rank, with no exchange of data.  Host checks that
every row and every expert is owned exactly once, and a world-size-2 gloo
run in which each rank computes its own shard of the oracle's products and
the gathered shards equal the unsharded product."""
import os
import sys
from pathlib import Path

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]
sys.path.insert(0, str(ROOT))
import workloads as wl  # noqa: E402


@pytest.mark.parametrize("M", [1, 127, 128, 129, 1000, 4096, 4096 * 3 + 5])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_row_shard_partitions_the_batch(M, world):
    owner = np.full(M, -1)
    for r in range(world):
        r0, r1 = wl.row_shard(M, world, r)
        assert 0 <= r0 <= r1 <= M
        if r1 > r0:  # whole tiles, the ragged tail last (ranks past the tile count get nothing)
            assert r0 % 128 == 0 and (r1 % 128 == 0 or r1 == M)
        assert np.all(owner[r0:r1] == -1)
        owner[r0:r1] = r
    assert np.all(owner >= 0)
    tiles = [-(-int(np.subtract(*wl.row_shard(M, world, r)[::-1])) // 128) for r in range(world)]
    assert max(tiles) - min(tiles) <= 1  # balanced to one tile


@pytest.mark.parametrize("E", [1, 7, 32, 256])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_expert_shard_partitions_the_experts(E, world):
    got = []
    for r in range(world):
        e0, e1 = wl.expert_shard(E, world, r)
        got.extend(range(e0, e1))
    assert got == list(range(E))


def test_shard_rejects_bad_rank():
    with pytest.raises(ValueError):
        wl.row_shard(128, 2, 2)
    with pytest.raises(ValueError):
        wl.expert_shard(4, 0, 0)


def test_dense_shards_share_the_layer():
    """Rank r > 0 draws its own tokens for the same layer: B and the
    per-channel magnitudes are rank 0's."""
    d0 = wl.dense_fprop(M=256, N=256, K=512)
    d1 = wl.dense_fprop(M=256, N=256, K=512, shard=1)
    assert np.array_equal(d0.b, d1.b) and not np.array_equal(d0.a, d1.a)
    assert d1.meta["shard"] == 1


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    import oracle
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # dense: this rank's row block of C = A B^T (quantize own rows, B replicated)
        d = wl.dense_fprop(M=300, N=256, K=512)
        r0, r1 = wl.row_shard(d.M, world, rank)
        qa, sa = oracle.quant_act_1x128(np.ascontiguousarray(d.a[r0:r1]))
        qb, sb = oracle.quant_w_128x128(d.b)
        c_local = torch.from_numpy(oracle.gemm_blockscaled(qa, sa, qb, sb))
        sizes = [wl.row_shard(d.M, world, r)[1] - wl.row_shard(d.M, world, r)[0] for r in range(world)]
        parts = [torch.zeros((n, d.N), dtype=torch.float64) for n in sizes]
        padded = max(sizes)
        buf = torch.zeros((padded, d.N), dtype=torch.float64)
        buf[:c_local.shape[0]] = c_local
        gathered = [torch.zeros_like(buf) for _ in range(world)]
        dist.all_gather(gathered, buf)
        dense = torch.cat([g[:n] for g, n in zip(gathered, sizes)]).numpy()
        # masked MoE: this rank's experts
        m = wl.moe_masked(E=4, cap=128, N=256, K=256, second=False)
        e0, e1 = wl.expert_shard(m.E, world, rank)
        qa3, sa3 = oracle.quant_act_1x128(np.ascontiguousarray(m.a[e0:e1].reshape(-1, 256)))
        qb3, sb3 = oracle.quant_w_128x128(np.ascontiguousarray(m.b[e0:e1]))
        local = oracle.grouped_masked(qa3.reshape(e1 - e0, 128, 256), sa3.reshape(e1 - e0, 128, 2), qb3, sb3,
                                      m.masked_m[e0:e1].astype(np.int32),
                                      out=np.zeros(((e1 - e0) * 128, 256)))
        mbuf = torch.zeros((2 * 128, 256), dtype=torch.float64)
        mbuf[:local.shape[0]] = torch.from_numpy(np.asarray(local, dtype=np.float64).reshape(-1, 256))
        mg = [torch.zeros_like(mbuf) for _ in range(world)]
        dist.all_gather(mg, mbuf)
        counts = [wl.expert_shard(m.E, world, r) for r in range(world)]
        moe = torch.cat([g[:(c1 - c0) * 128] for g, (c0, c1) in zip(mg, counts)]).numpy()
        q.put((rank, dense, moe))
    finally:
        dist.destroy_process_group()


def test_shards_concatenate_to_the_full_product_gloo_world2():
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29700 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        rank, dense, moe = q.get(timeout=300)
        res[rank] = (dense, moe)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    d = wl.dense_fprop(M=300, N=256, K=512)
    qa, sa = oracle.quant_act_1x128(d.a)
    qb, sb = oracle.quant_w_128x128(d.b)
    full = oracle.gemm_blockscaled(qa, sa, qb, sb)
    m = wl.moe_masked(E=4, cap=128, N=256, K=256, second=False)
    qa3, sa3 = oracle.quant_act_1x128(np.ascontiguousarray(m.a.reshape(-1, 256)))
    qb3, sb3 = oracle.quant_w_128x128(m.b)
    full_moe = oracle.grouped_masked(qa3.reshape(4, 128, 256), sa3.reshape(4, 128, 2), qb3, sb3,
                                     m.masked_m.astype(np.int32), out=np.zeros((4 * 128, 256)))
    for rank in range(2):
        dense, moe = res[rank]
        assert np.array_equal(dense, full)  # each row computed once, by its owner, identically
        assert np.array_equal(moe, np.asarray(full_moe).reshape(-1, 256))
