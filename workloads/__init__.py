"""Seeded synthetic inputs for the fine-grained FP8 quantization + GEMM path.

This module holds random draws and input layout only -- none of the method's
arithmetic (no scaling, no E4M3 encoding, no products).  It is the one module
that both the CPU oracle side and the CUDA side of the tests and the benchmark
take their inputs from.  Every tensor is produced as bf16 *bit patterns*
(``numpy.uint16``) so the same bytes go to the oracle and to the GPU.

Workloads (shapes and distributions of the MoE/dense Linear layers the pages
discuss; all seeds are numpy PCG64):

* ``tiny_dense``      A 128x512 N(0,1) with 0.1% of entries scaled x100, B 256x512 N(0,1); seed 0.
* ``dense_fprop``     A 4096x7168 z[m,k]*exp(g[k]) (per-channel log-normal, sigma 1) plus 0.01%
                      entries set to +-200; B 7168x7168 N(0, 0.02^2); seed 1.
* ``long_k``          A 2048x16384, B 2048x16384, both U[-1,1] + 0.5; seed 2.
* ``moe_contiguous``  4096 tokens, top-8 of 32 experts with Zipf(1.1) expert popularity, rows of each
                      expert padded to a multiple of 128 (pad rows zero); A N(0,1) [M_tot,7168];
                      B [32,4096,7168] N(0,0.02^2); m_indices = expert of each 128-row block; seed 3.
* ``moe_masked``      32 experts x capacity 256, valid counts uniform on {0..256}; A [32,256,7168]
                      N(0,1), B1 [32,4096,7168]; second GEMM A2 [32,256,2048] N(0,1), B2
                      [32,7168,2048]; weights N(0,0.02^2); seed 4.
* ``dense_wgrad``     the weight gradient of the dense_fprop layer, dW = dY^T X over 4096 tokens:
                      X is dense_fprop's A (seed 1); dY [4096,7168] z[m,n]*exp(g[n]) (per-channel
                      log-normal, sigma 1), seed 5.

Every generator takes size overrides so the tests can draw the same
distributions at sizes the oracle finishes in seconds.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

TILE = 128


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 array -> bf16 bit patterns (uint16), round-to-nearest-even.

    Input preparation only: the generators draw in float32 and store bf16.
    Non-finite values are not produced by any generator here."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    # finite inputs: the largest pattern, 0xFF7FFFFF, plus 0x8000 stays below 2^32
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact widening)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal_bf16(rng: np.random.Generator, shape, std: float = 1.0, chunk_rows: int = 4096) -> np.ndarray:
    """N(0, std^2) bf16 bits, drawn in row chunks to bound host memory."""
    shape = tuple(int(s) for s in shape)
    out = np.empty(shape, dtype=np.uint16)
    flat = out.reshape(-1, shape[-1]) if len(shape) > 1 else out.reshape(1, -1)
    for r0 in range(0, flat.shape[0], chunk_rows):
        r1 = min(flat.shape[0], r0 + chunk_rows)
        z = rng.standard_normal((r1 - r0, flat.shape[1]), dtype=np.float32)
        if std != 1.0:
            z *= np.float32(std)
        flat[r0:r1] = bf16_bits(z)
    return out


@dataclass
class Dense:
    name: str
    a: np.ndarray  # [M,K] bf16 bits
    b: np.ndarray  # [N,K] bf16 bits
    meta: dict = field(default_factory=dict)

    @property
    def M(self):
        return self.a.shape[0]

    @property
    def N(self):
        return self.b.shape[0]

    @property
    def K(self):
        return self.a.shape[1]

    @property
    def flops(self):
        return 2.0 * self.M * self.N * self.K


def tiny_dense(seed: int = 0, M: int = 128, N: int = 256, K: int = 512, outlier_frac: float = 1e-3,
               outlier_mult: float = 100.0) -> Dense:
    rng = np.random.default_rng(seed)
    a = rng.standard_normal((M, K), dtype=np.float32)
    n_out = int(round(outlier_frac * M * K))
    idx = rng.choice(M * K, size=n_out, replace=False)
    a.reshape(-1)[idx] *= np.float32(outlier_mult)
    b = rng.standard_normal((N, K), dtype=np.float32)
    return Dense("tiny_dense", bf16_bits(a), bf16_bits(b), {"seed": seed, "outliers": n_out})


def dense_fprop(seed: int = 1, M: int = 4096, N: int = 7168, K: int = 7168, outlier_frac: float = 1e-4,
                outlier_value: float = 200.0, w_std: float = 0.02, shard: int = 0) -> Dense:
    """``shard`` r > 0 draws the r-th M-row block of a larger token batch: the
    same layer (per-channel magnitudes and weight B, both from ``seed``), its
    own tokens (seeded by (seed, r)).  Shard 0 is the single-GPU workload."""
    if shard:
        base = dense_fprop(seed, M=TILE, N=N, K=K, outlier_frac=0.0, w_std=w_std)
        b_bits = dense_fprop(seed, M=M, N=N, K=K, outlier_frac=outlier_frac, outlier_value=outlier_value,
                             w_std=w_std).b
        rng = np.random.default_rng([seed, shard])
        chan = base.meta["chan"]
        a = rng.standard_normal((M, K), dtype=np.float32)
        a *= chan[None, :]
        n_out = int(round(outlier_frac * M * K))
        idx = rng.choice(M * K, size=n_out, replace=False)
        signs = np.where(rng.random(n_out) < 0.5, -1.0, 1.0).astype(np.float32)
        a.reshape(-1)[idx] = np.float32(outlier_value) * signs
        return Dense("dense_fprop", bf16_bits(a), b_bits, {"seed": seed, "shard": shard, "outliers": n_out})
    rng = np.random.default_rng(seed)
    g = rng.standard_normal(K, dtype=np.float32)
    chan = np.exp(g).astype(np.float32)  # per-channel log-normal magnitude, sigma = 1
    a = rng.standard_normal((M, K), dtype=np.float32)
    a *= chan[None, :]
    n_out = int(round(outlier_frac * M * K))
    idx = rng.choice(M * K, size=n_out, replace=False)
    signs = np.where(rng.random(n_out) < 0.5, -1.0, 1.0).astype(np.float32)
    a.reshape(-1)[idx] = np.float32(outlier_value) * signs
    a_bits = bf16_bits(a)
    del a
    b_bits = _normal_bf16(rng, (N, K), w_std)
    return Dense("dense_fprop", a_bits, b_bits, {"seed": seed, "outliers": n_out, "chan": chan})


@dataclass
class Wgrad:
    name: str
    dy: np.ndarray  # [M,N] bf16 bits (tokens x output channels)
    x: np.ndarray   # [M,K] bf16 bits (tokens x input channels)
    meta: dict = field(default_factory=dict)

    @property
    def M(self):
        return self.x.shape[0]

    @property
    def N(self):
        return self.dy.shape[1]

    @property
    def K(self):
        return self.x.shape[1]

    @property
    def flops(self):
        return 2.0 * self.M * self.N * self.K


def dense_wgrad(seed: int = 5, M: int = 4096, N: int = 7168, K: int = 7168) -> Wgrad:
    x = dense_fprop(M=M, N=128, K=K).a
    rng = np.random.default_rng(seed)
    chan = np.exp(rng.standard_normal(N, dtype=np.float32)).astype(np.float32)
    dy = np.empty((M, N), dtype=np.uint16)
    for r0 in range(0, M, 1024):
        z = rng.standard_normal((min(M, r0 + 1024) - r0, N), dtype=np.float32)
        z *= chan[None, :]
        dy[r0:r0 + z.shape[0]] = bf16_bits(z)
    return Wgrad("dense_wgrad", dy, x, {"seed": seed, "x_seed": 1})


def long_k(seed: int = 2, M: int = 2048, N: int = 2048, K: int = 16384, shift: float = 0.5, shard: int = 0) -> Dense:
    """``shard`` r > 0: the r-th M-row block of a larger batch (same B, own rows)."""
    rng = np.random.default_rng(seed)
    a = rng.uniform(-1.0, 1.0, size=(M, K)).astype(np.float32) + np.float32(shift)
    b = rng.uniform(-1.0, 1.0, size=(N, K)).astype(np.float32) + np.float32(shift)
    if shard:
        a = np.random.default_rng([seed, shard]).uniform(-1.0, 1.0, size=(M, K)).astype(np.float32) + np.float32(shift)
    return Dense("long_k", bf16_bits(a), bf16_bits(b), {"seed": seed, "shard": shard})


@dataclass
class Contiguous:
    name: str
    a: np.ndarray          # [M_tot,K] bf16 bits (pad rows zero)
    b: np.ndarray          # [E,N,K] bf16 bits
    m_indices: np.ndarray  # [M_tot/128] int32
    counts: np.ndarray     # [E] valid rows per expert
    meta: dict = field(default_factory=dict)

    @property
    def M_tot(self):
        return self.a.shape[0]

    @property
    def E(self):
        return self.b.shape[0]

    @property
    def N(self):
        return self.b.shape[1]

    @property
    def K(self):
        return self.a.shape[1]

    @property
    def flops(self):
        """Algorithmic FLOPs: valid (unpadded) rows only."""
        return 2.0 * float(self.counts.sum()) * self.N * self.K

    @property
    def flops_padded(self):
        return 2.0 * self.M_tot * self.N * self.K


def zipf_topk_counts(rng: np.random.Generator, tokens: int, E: int, topk: int, alpha: float) -> np.ndarray:
    """Rows per expert for ``tokens`` tokens each routed to ``topk`` distinct
    experts.  Expert popularity p_e ~ rank_e^-alpha over a random permutation of
    ranks; each token samples ``topk`` experts without replacement
    (Gumbel-top-k on log p)."""
    ranks = rng.permutation(E) + 1
    logp = -alpha * np.log(ranks.astype(np.float64))
    g = rng.gumbel(size=(tokens, E))
    chosen = np.argsort(-(logp[None, :] + g), axis=1)[:, :topk]
    return np.bincount(chosen.reshape(-1), minlength=E).astype(np.int64)


def device_normal_bf16(shape, std: float, seed: int, device):
    """N(0, std^2) as a bf16 tensor drawn on a CUDA device with torch's seeded
    Philox generator (float32 draws, rounded to bf16 to nearest even).  The
    same distribution as the host draws, other values: for timing runs of the
    large MoE weights, where the host generator would take a minute."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    z = torch.randn(tuple(int(v) for v in shape), generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        z.mul_(std)
    return z.to(torch.bfloat16)


def moe_contiguous(seed: int = 3, tokens: int = 4096, topk: int = 8, E: int = 32, N: int = 4096, K: int = 7168,
                   alpha: float = 1.1, w_std: float = 0.02, device=None, shard: int = 0) -> Contiguous:
    """With ``device`` given, ``a`` and ``b`` are bf16 tensors drawn on that
    device (device_normal_bf16, seeds derived from ``seed``); the routing
    (counts, m_indices) is the host draw either way.  ``shard`` r > 0 draws
    the r-th rank's experts of an expert-parallel layer E times the ranks
    wide: its own tokens' rows and its own expert weights, seeded by
    (seed, r)."""
    rng = np.random.default_rng([seed, shard] if shard else seed)
    dseed = seed * 1000 + 100000 * shard
    counts = zipf_topk_counts(rng, tokens, E, topk, alpha)
    padded = (counts + TILE - 1) // TILE * TILE
    M_tot = int(padded.sum())
    m_indices = np.empty(M_tot // TILE, dtype=np.int32)
    if device is not None:
        import torch
        a = torch.zeros((M_tot, K), dtype=torch.bfloat16, device=device)
    else:
        a = np.zeros((M_tot, K), dtype=np.uint16)
    r = 0
    for e in range(E):
        c, p = int(counts[e]), int(padded[e])
        if c:
            if device is not None:
                a[r:r + c] = device_normal_bf16((c, K), 1.0, dseed + e, device)
            else:
                a[r:r + c] = _normal_bf16(rng, (c, K))
        m_indices[r // TILE:(r + p) // TILE] = e
        r += p
    if device is not None:
        b = device_normal_bf16((E, N, K), w_std, dseed + 999, device)
    else:
        b = _normal_bf16(rng, (E, N, K), w_std)
    return Contiguous("moe_contiguous", a, b, m_indices, counts,
                      {"seed": seed, "shard": shard, "tokens": tokens, "topk": topk,
                       "draws": "device" if device is not None else "host"})


@dataclass
class Masked:
    name: str
    a: np.ndarray         # [E,cap,K] bf16 bits
    b: np.ndarray         # [E,N,K] bf16 bits
    masked_m: np.ndarray  # [E] int32
    a2: np.ndarray | None = None  # second GEMM [E,cap,K2]
    b2: np.ndarray | None = None  # [E,N2,K2]
    meta: dict = field(default_factory=dict)

    @property
    def E(self):
        return self.a.shape[0]

    @property
    def cap(self):
        return self.a.shape[1]

    def flops(self, second: bool = False):
        b = self.b2 if second else self.b
        return 2.0 * float(self.masked_m.sum()) * b.shape[1] * b.shape[2]


def moe_masked(seed: int = 4, E: int = 32, cap: int = 256, N: int = 4096, K: int = 7168, N2: int = 7168,
               K2: int = 2048, w_std: float = 0.02, second: bool = True, device=None, shard: int = 0) -> Masked:
    """With ``device`` given, the activations and weights are bf16 tensors
    drawn on that device (device_normal_bf16); masked_m is the host draw
    either way.  ``shard`` r > 0: the r-th rank's experts of an
    expert-parallel layer, seeded by (seed, r)."""
    rng = np.random.default_rng([seed, shard] if shard else seed)
    masked_m = rng.integers(0, cap, size=E, endpoint=True).astype(np.int32)
    if device is not None:
        def draw(shape, std, k):
            return device_normal_bf16(shape, std, seed * 1000 + 100000 * shard + k, device)
    else:
        def draw(shape, std, k):
            return _normal_bf16(rng, shape, std)
    a = draw((E, cap, K), 1.0, 0)
    b = draw((E, N, K), w_std, 1)
    a2 = b2 = None
    if second:
        a2 = draw((E, cap, K2), 1.0, 2)
        b2 = draw((E, N2, K2), w_std, 3)
    return Masked("moe_masked", a, b, masked_m, a2, b2,
                  {"seed": seed, "shard": shard, "draws": "device" if device is not None else "host"})


def parity_rows(rng: np.random.Generator, M: int, per_tile: int = 2, tile: int = TILE) -> np.ndarray:
    """Seeded sample of row indices: ``per_tile`` rows from every 128-row tile
    (first and last row of the tile always included, so ragged tails count)."""
    rows = []
    for t0 in range(0, M, tile):
        t1 = min(M, t0 + tile)
        pick = {t0, t1 - 1}
        extra = max(0, per_tile - len(pick))
        if extra and t1 - t0 > 2:
            pick.update(int(v) for v in rng.choice(np.arange(t0 + 1, t1 - 1), size=min(extra, t1 - t0 - 2),
                                                     replace=False))
        rows.extend(sorted(pick))
    return np.asarray(rows, dtype=np.int64)


def row_shard(M: int, world: int, rank: int, tile: int = TILE) -> tuple[int, int]:
    """Rows [start, stop) of an M-row batch owned by ``rank`` of ``world``:
    contiguous runs of whole 128-row tiles, as even as the tile count allows
    (the first M_tiles % world ranks take one tile more); the last rank's run
    ends at M, ragged tail included.  Every row belongs to exactly one rank."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank %d of world %d" % (rank, world))
    tiles = -(-M // tile)
    base, extra = divmod(tiles, world)
    t0 = rank * base + min(rank, extra)
    t1 = t0 + base + (1 if rank < extra else 0)
    return min(M, t0 * tile), min(M, t1 * tile)


def expert_shard(E: int, world: int, rank: int) -> tuple[int, int]:
    """Experts [e0, e1) owned by ``rank`` (expert parallelism): contiguous,
    as even as E allows; every expert belongs to exactly one rank."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank %d of world %d" % (rank, world))
    base, extra = divmod(E, world)
    e0 = rank * base + min(rank, extra)
    return e0, e0 + base + (1 if rank < extra else 0)


def quad_rows(rng: np.random.Generator, M: int, tile: int = TILE, quad: int = 32) -> np.ndarray:
    """Seeded sample of row indices that reaches every 32-row quad of every
    128-row tile: the tile's first and last row, plus one seeded row inside
    each quad that holds valid rows (a ragged last tile only has the quads
    below M).  The GEMM's epilogue assigns each quad of a tile to its own
    warps, so every warp's rows are compared on every tile."""
    rows = []
    for t0 in range(0, M, tile):
        t1 = min(M, t0 + tile)
        pick = {t0, t1 - 1}
        for q0 in range(t0, t1, quad):
            q1 = min(t1, q0 + quad)
            pick.add(int(rng.integers(q0, q1)))
        rows.extend(sorted(pick))
    return np.asarray(rows, dtype=np.int64)


CONFIGS = {
    "tiny_dense": tiny_dense,
    "dense_fprop": dense_fprop,
    "long_k": long_k,
    "moe_contiguous": moe_contiguous,
    "moe_masked": moe_masked,
    "dense_wgrad": dense_wgrad,
}
