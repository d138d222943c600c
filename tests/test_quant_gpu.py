"""GPU quantizers vs the oracle: E4M3 codes and scales must match bit for bit.

Covers the hand-computed worked examples, edge tensors (zeros, -0, exact
ties, E4M3 subnormals, bf16 subnormals, +-448 boundaries, huge values),
ragged row counts, and every workload's full-size tensors.
"""
import numpy as np
import pytest
import torch

import oracle
import fp8_fine_grained_quant_b200 as fq
import workloads as wl
from conftest import golden_lines, hexfloat
from parity import bytes_of, to_torch_bf16

pytestmark = pytest.mark.gpu
TILE = 128


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def gpu_act(bits, dev):
    x = to_torch_bf16(bits, dev)
    q, s = fq.fp8_quant_act_1x128(x)
    torch.cuda.synchronize(dev)
    assert fq.get_device_error(device=dev) == fq.OK
    return bytes_of(q), s.cpu().numpy()


def gpu_w(bits, dev):
    w = to_torch_bf16(bits, dev)
    q, s = fq.fp8_quant_w_128x128(w)
    torch.cuda.synchronize(dev)
    return bytes_of(q).reshape(bits.shape), s.cpu().numpy()


def assert_act_exact(bits, dev):
    q, s = gpu_act(bits, dev)
    oq, os_ = oracle.quant_act_1x128(bits)
    assert np.array_equal(s.reshape(os_.shape).view(np.uint32), os_.view(np.uint32)), \
        np.argwhere(s.reshape(os_.shape).view(np.uint32) != os_.view(np.uint32))[:5]
    bad = np.argwhere(q.reshape(oq.shape) != oq)
    assert bad.size == 0, (bad[:5], q.reshape(oq.shape)[tuple(bad[0])], oq[tuple(bad[0])])


def assert_w_exact(bits, dev):
    q, s = gpu_w(bits, dev)
    oq, os_ = oracle.quant_w_128x128(bits)
    assert np.array_equal(s.reshape(os_.shape).view(np.uint32), os_.view(np.uint32))
    bad = np.argwhere(q.reshape(oq.shape) != oq)
    assert bad.size == 0, bad[:5]


def test_worked_examples(dev):
    rows = {}
    for tok in golden_lines("quant_worked_examples.txt"):
        if tok[0] in ("act", "act2") and tok[1] != "K":
            rows.setdefault(tok[0], []).append((int(tok[1]), hexfloat(tok[2]), int(tok[3], 16)))
    for kind, K in (("act", 384), ("act2", 128)):
        x = np.zeros((1, K), dtype=np.float32)
        expect = np.zeros(K, dtype=np.uint8)
        for k, v, code in rows[kind]:
            x[0, k] = v
            expect[k] = code
        q, _ = gpu_act(wl.bf16_bits(x), dev)
        assert np.array_equal(q.reshape(-1), expect), kind


def _edge_tile_values():
    """One 128-wide tile per row, each exercising a boundary of the encoder."""
    v = []
    ramp = np.arange(128, dtype=np.float32)
    v.append(np.zeros(128, np.float32))                          # zero tile
    v.append(-np.zeros(128, np.float32))                         # -0 tile
    v.append(np.full(128, 448.0, np.float32) * np.where(ramp % 2, -1, 1))  # +-448, s = 1
    t = (ramp - 64) * np.float32(3.5)                            # many exact ties after scaling
    t[0] = 448.0
    v.append(t)
    v.append(np.float32(2.0) ** -(ramp % 30 + 1) * np.where(ramp % 3, 1, -1))  # wide dynamic range
    v.append(np.full(128, np.float32(1e-38)) * (ramp + 1))       # near-subnormal scale
    sub = np.full(128, np.float32(2.0 ** -133)) * (ramp % 7)     # bf16 subnormals
    v.append(sub)
    big = np.full(128, np.float32(3.0e38)) * np.where(ramp % 2, -1, 1)
    big[5] = 1.0
    v.append(big)
    mix = np.float32(56.0) * np.float32(2.0) ** -(ramp % 20)     # s = 1/8, codes cover subnormals
    v.append(mix)
    return np.stack(v)


def test_edge_tiles(dev):
    bits = wl.bf16_bits(_edge_tile_values())
    assert_act_exact(bits, dev)
    # as weights: replicate the pattern into a 128 x (9*128) block row
    w = np.repeat(bits.reshape(1, -1), 128, axis=0)
    assert_w_exact(np.ascontiguousarray(w), dev)


@pytest.mark.parametrize("M,K", [(1, 128), (3, 256), (129, 384), (300, 1024), (2048, 128), (7, 7168)])
def test_act_random_shapes(dev, M, K):
    rng = np.random.default_rng(M * 131 + K)
    x = rng.standard_normal((M, K)).astype(np.float32) * np.exp(rng.uniform(-8, 8, size=(M, 1))).astype(np.float32)
    x.reshape(-1)[rng.choice(M * K, size=max(1, M * K // 1000), replace=False)] *= 100
    assert_act_exact(wl.bf16_bits(x), dev)


@pytest.mark.parametrize("G,N,K", [(1, 128, 128), (1, 256, 640), (3, 384, 256), (2, 1024, 2048)])
def test_w_random_shapes(dev, G, N, K):
    rng = np.random.default_rng(G * 7 + N + K)
    w = (0.02 * rng.standard_normal((G, N, K))).astype(np.float32)
    w[:, ::97, ::89] *= 50
    assert_w_exact(wl.bf16_bits(w), dev)


def test_zero_sizes_are_noops(dev):
    x = torch.zeros((0, 256), dtype=torch.bfloat16, device=dev)
    q, s = fq.fp8_quant_act_1x128(x)
    assert q.shape == (0, 256) and s.shape == (0, 2)


@pytest.mark.parametrize("name", ["tiny_dense", "dense_fprop", "long_k"])
def test_dense_workloads_full(dev, name):
    d = wl.CONFIGS[name]()
    assert_act_exact(d.a, dev)
    assert_w_exact(d.b, dev)


def test_moe_contiguous_full(dev):
    d = wl.moe_contiguous()
    assert_act_exact(d.a, dev)
    assert_w_exact(d.b, dev)


def test_moe_masked_full(dev):
    d = wl.moe_masked()
    assert_act_exact(d.a.reshape(-1, d.a.shape[-1]), dev)
    assert_w_exact(d.b, dev)
    assert_act_exact(d.a2.reshape(-1, d.a2.shape[-1]), dev)
    assert_w_exact(d.b2, dev)


def _near_midpoint_tiles(seed=17, n_scales=400):
    """Tiles whose quotients x/s land within a few binary32 ulps of an E4M3
    rounding midpoint (where a product with 1/s could round differently from
    the quotient).  Selection only: the expected codes come from the oracle."""
    rng = np.random.default_rng(seed)
    pos = np.arange(1, 0x7F80, dtype=np.uint16)  # all positive finite bf16
    xs_all = wl.bf16_to_f32(pos)
    tiles = []
    for _ in range(n_scales):
        amax = wl.bf16_to_f32(wl.bf16_bits(np.float32(np.exp(rng.uniform(-30, 30))))).reshape(-1)[0]
        s = np.float32(amax / np.float32(448.0))
        if s == 0 or s < np.float32(2.0 ** -125):
            continue
        xs = xs_all[xs_all <= amax]
        qt = (xs / s).astype(np.float32)
        b = qt.view(np.uint32)
        normal = qt >= np.float32(2.0 ** -6)
        rem = (b & np.uint32(0xFFFFF)).astype(np.int64) - 0x80000
        near = normal & (np.abs(rem) <= 64)
        t = qt * np.float32(512.0)
        near |= (~normal) & (np.abs(t - np.trunc(t) - 0.5) <= 2.0 ** -16)
        pick = xs[near][:127]
        if pick.size == 0:
            continue
        row = np.zeros(128, dtype=np.float32)
        row[0] = amax
        row[1:1 + pick.size] = pick * np.where(rng.random(pick.size) < 0.5, -1, 1)
        tiles.append(row)
    return np.stack(tiles)


def test_quotients_near_e4m3_midpoints(dev):
    x = _near_midpoint_tiles()
    assert x.shape[0] > 100
    bits = wl.bf16_bits(x)
    assert_act_exact(bits, dev)
    # the same values as 128x128 weight blocks (one scale per block of 128 such rows)
    rows = (x.shape[0] // 128) * 128
    if rows:
        assert_w_exact(np.ascontiguousarray(bits[:rows]), dev)


def _tiles_with_every_amax(stride=1, seed=7):
    """One 128-element group per finite non-negative bf16 value a (every
    `stride`-th one): element 0 is a, the rest are random values of magnitude
    at most a, either sign.  Returns the bf16 bits, [groups, 128]."""
    amax_bits = np.arange(0, 0x7F80, stride, dtype=np.uint32)
    a = (amax_bits << 16).view(np.float32)
    rng = np.random.default_rng(seed)
    u = rng.random((a.size, TILE), dtype=np.float32)
    sign = np.where(rng.random((a.size, TILE)) < 0.5, -1.0, 1.0).astype(np.float32)
    x = wl.bf16_bits(a[:, None] * u * sign)
    x[:, 0] = amax_bits.astype(np.uint16)
    return x


def test_every_bf16_amax_act(dev):
    """All 32640 finite non-negative bf16 amax values, one tile each: the
    division-free scale and the codes must equal the oracle's IEEE results."""
    x = _tiles_with_every_amax()
    assert x.shape[0] == 255 * 128
    assert_act_exact(x.reshape(255, 128 * TILE), dev)


def test_every_16th_bf16_amax_w(dev):
    """Every 16th bf16 amax value, one 128x128 weight block each."""
    groups = _tiles_with_every_amax(stride=16, seed=8)   # 2040 groups of 128
    nb = groups.shape[0]
    rng = np.random.default_rng(9)
    blocks = np.empty((nb, TILE, TILE), dtype=np.uint16)
    # each block: the group as its first row, the other rows a shuffled copy
    # scaled down by a power of two (exact in bf16 unless it underflows)
    f = wl.bf16_to_f32(groups)
    for i in range(nb):
        rows = np.stack([rng.permutation(f[i]) for _ in range(TILE - 1)]) * np.float32(0.5)
        blocks[i, 0] = groups[i]
        blocks[i, 1:] = wl.bf16_bits(rows)
    w = blocks.reshape(nb * TILE, TILE)   # G = 1, N = 128 * nb, K = 128
    assert_w_exact(w, dev)


# --------------------------------------------------------------------------- power-of-two (UE8M0) scales
@pytest.mark.parametrize("M,K", [(300, 384), (1, 128), (4096, 7168)])
def test_ue8m0_act_matches_oracle(dev, M, K):
    rng = np.random.default_rng(M + K)
    x = wl.bf16_bits((rng.standard_normal((M, K)) * np.exp(rng.standard_normal(K))).astype(np.float32))
    x[0, :] = 0
    q, s = fq.fp8_quant_act_1x128_ue8m0(to_torch_bf16(x, dev))
    torch.cuda.synchronize(dev)
    oq, os_ = oracle.quant_act_1x128_ue8m0(x)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), os_.view(np.uint32))
    assert np.array_equal(bytes_of(q).reshape(M, K), oq)


def test_ue8m0_every_bf16_amax(dev):
    x = _tiles_with_every_amax()
    x2 = x.reshape(255, 128 * TILE)
    q, s = fq.fp8_quant_act_1x128_ue8m0(to_torch_bf16(x2, dev))
    torch.cuda.synchronize(dev)
    oq, os_ = oracle.quant_act_1x128_ue8m0(x2)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), os_.view(np.uint32))
    assert np.array_equal(bytes_of(q).reshape(oq.shape), oq)


@pytest.mark.parametrize("G,N,K", [(1, 256, 384), (3, 128, 256)])
def test_ue8m0_w_matches_oracle(dev, G, N, K):
    rng = np.random.default_rng(G + N + K)
    w = wl.bf16_bits((0.02 * rng.standard_normal((G, N, K))).astype(np.float32))
    q, s = fq.fp8_quant_w_128x128_ue8m0(to_torch_bf16(w, dev))
    torch.cuda.synchronize(dev)
    oq, os_ = oracle.quant_w_128x128_ue8m0(w)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), os_.view(np.uint32))
    assert np.array_equal(bytes_of(q).reshape(oq.shape), oq)


# ------------------------------------------------------------------ both operands in one launch
def _fused_exact(a_bits, w_bits, dev):
    x = to_torch_bf16(a_bits, dev)
    w = to_torch_bf16(w_bits, dev)
    (qa, sa), (qw, sw) = fq.fp8_quant_act_w(x, w)
    torch.cuda.synchronize(dev)
    assert fq.get_device_error(device=dev) == fq.OK
    if a_bits.size:
        oq, os_ = oracle.quant_act_1x128(a_bits)
        assert np.array_equal(sa.cpu().numpy().reshape(os_.shape).view(np.uint32), os_.view(np.uint32))
        assert np.array_equal(bytes_of(qa).reshape(oq.shape), oq)
    if w_bits.size:
        oq, os_ = oracle.quant_w_128x128(w_bits)
        assert np.array_equal(sw.cpu().numpy().reshape(os_.shape).view(np.uint32), os_.view(np.uint32))
        assert np.array_equal(bytes_of(qw).reshape(oq.shape), oq)
    return (qa, sa), (qw, sw)


@pytest.mark.parametrize("M,K,Gw,N,Kw", [
    (300, 384, 1, 256, 640),     # 900 tiles: a partial last activation unit
    (1, 128, 3, 128, 128),       # one tile, batched weights
    (4097, 1024, 2, 384, 256),   # ragged rows, more units than SMs
])
def test_fused_operands_exact(dev, M, K, Gw, N, Kw):
    rng = np.random.default_rng(M + K + N)
    a = wl.bf16_bits((rng.standard_normal((M, K)) * np.exp(rng.standard_normal(K))).astype(np.float32))
    w = wl.bf16_bits((0.02 * rng.standard_normal((Gw, N, Kw))).astype(np.float32))
    _fused_exact(a, w if Gw > 1 else w[0], dev)


def test_fused_operands_equal_the_separate_kernels_dense_fprop(dev):
    """dense_fprop in full: the fused launch gives the bytes of the two
    separate quantizers, which are bit-exact against the oracle."""
    d = wl.dense_fprop()
    (qa, sa), (qw, sw) = _fused_exact(d.a, d.b, dev)
    qa2, sa2 = fq.fp8_quant_act_1x128(to_torch_bf16(d.a, dev))
    qw2, sw2 = fq.fp8_quant_w_128x128(to_torch_bf16(d.b, dev))
    torch.cuda.synchronize(dev)
    assert torch.equal(qa.view(torch.uint8), qa2.view(torch.uint8)) and torch.equal(sa, sa2)
    assert torch.equal(qw.view(torch.uint8), qw2.view(torch.uint8)) and torch.equal(sw, sw2)


def test_fused_operands_one_side_empty(dev):
    rng = np.random.default_rng(9)
    a = wl.bf16_bits(rng.standard_normal((64, 256)).astype(np.float32))
    w = wl.bf16_bits(rng.standard_normal((128, 256)).astype(np.float32))
    x = to_torch_bf16(a, dev)
    ww = to_torch_bf16(w, dev)
    (qa, sa), _ = fq.fp8_quant_act_w(x, torch.empty((0, 128, 256), dtype=torch.bfloat16, device=dev))
    torch.cuda.synchronize(dev)
    oq, os_ = oracle.quant_act_1x128(a)
    assert np.array_equal(bytes_of(qa).reshape(oq.shape), oq)
    _, (qw, sw) = fq.fp8_quant_act_w(torch.empty((0, 128), dtype=torch.bfloat16, device=dev), ww)
    torch.cuda.synchronize(dev)
    oq, os_ = oracle.quant_w_128x128(w)
    assert np.array_equal(bytes_of(qw).reshape(oq.shape), oq)
    assert fq.get_device_error(device=dev) == fq.OK
