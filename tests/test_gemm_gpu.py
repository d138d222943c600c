"""GPU block-scaled GEMMs vs the oracle's float64 dequantized-input product.

Tolerance (written here, from the target): max |C - C_ref| <= 1e-2 * rms(C_ref)
and max relative error <= 2e-3 over elements with |C_ref| >= 0.1 * rms(C_ref)
(see parity.py).  The oracle quantizes the same bf16 inputs itself; nothing it
compares against comes from the GPU.  Small shapes are compared in full
(several tiles, ragged tails), among them shapes with more than twice as many
output tiles as the B200 has SMs, so every persistent CTA carries its state
(accumulator reset, scale-ring slot, barrier phases) over several tiles.
Full-size workloads are compared on a seeded row sample that reaches every
32-row quad of every 128-row tile (the rows of each epilogue warp), every
expert and all N columns.
"""
import numpy as np
import pytest
import torch

import oracle
import fp8_fine_grained_quant_b200 as fq
import workloads as wl
from parity import assert_gemm_close, bf16_bits_of, to_torch_bf16

pytestmark = pytest.mark.gpu
TILE = 128


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _quantize_both(a_bits, b_bits, dev):
    """GPU quantization (for the GPU GEMM) and oracle quantization (for the
    reference).  The quantizer tests establish that both are identical."""
    a = to_torch_bf16(a_bits.reshape(-1, a_bits.shape[-1]), dev)
    b = to_torch_bf16(b_bits, dev)
    qa, sa = fq.fp8_quant_act_1x128(a)
    qb, sb = fq.fp8_quant_w_128x128(b)
    oqa, osa = oracle.quant_act_1x128(np.ascontiguousarray(a_bits.reshape(-1, a_bits.shape[-1])))
    oqb, osb = oracle.quant_w_128x128(b_bits)
    return (qa, sa, qb, sb), (oqa, osa, oqb, osb)


def _finish(dev):
    torch.cuda.synchronize(dev)
    assert fq.get_device_error(device=dev) == fq.OK


@pytest.mark.parametrize("M,N,K", [
    (128, 256, 512),    # one tile
    (1, 128, 128),      # single row, single slab
    (300, 384, 640),    # ragged M, N = 3 weight blocks
    (257, 512, 1024),
    (129, 2048, 256),
    (64, 7168, 384),    # wide N
    (640, 128, 2048),   # N = one block
])
def test_dense_small_full(dev, M, N, K):
    rng = np.random.default_rng(M + 3 * N + 7 * K)
    a = rng.standard_normal((M, K)).astype(np.float32) * np.exp(rng.standard_normal(K)).astype(np.float32)
    b = (0.02 * rng.standard_normal((N, K))).astype(np.float32)
    (qa, sa, qb, sb), (oqa, osa, oqb, osb) = _quantize_both(wl.bf16_bits(a), wl.bf16_bits(b), dev)
    c = fq.fp8_gemm_blockscaled(qa, sa, qb, sb)
    _finish(dev)
    ref = oracle.gemm_blockscaled(oqa, osa, oqb, osb)
    assert_gemm_close(bf16_bits_of(c), ref, "dense %dx%dx%d" % (M, N, K))


def _misaligned_copy(t):
    """Same values, at an address 4 bytes past a 16-byte boundary."""
    buf = torch.empty(t.numel() + 1, dtype=t.dtype, device=t.device)
    view = buf[1:].view(t.shape)
    view.copy_(t)
    assert view.data_ptr() % 16 == 4
    return view


@pytest.mark.parametrize("M,N,K", [(257, 512, 1024), (128, 384, 2048)])
def test_scale_staging_paths_agree(dev, M, N, K):
    """K % 512 == 0 with 16-byte-aligned scales stages the scales through
    shared memory with the operands; unaligned scales take the global-load
    path.  Both must give the same bits (and match the oracle)."""
    rng = np.random.default_rng(M + N + K)
    a = rng.standard_normal((M, K)).astype(np.float32) * np.exp(rng.standard_normal(K)).astype(np.float32)
    b = (0.02 * rng.standard_normal((N, K))).astype(np.float32)
    (qa, sa, qb, sb), (oqa, osa, oqb, osb) = _quantize_both(wl.bf16_bits(a), wl.bf16_bits(b), dev)
    staged = fq.fp8_gemm_blockscaled(qa, sa, qb, sb)
    loaded = fq.fp8_gemm_blockscaled(qa, _misaligned_copy(sa), qb, _misaligned_copy(sb))
    _finish(dev)
    assert torch.equal(staged.view(torch.int16), loaded.view(torch.int16))
    assert_gemm_close(bf16_bits_of(staged), oracle.gemm_blockscaled(oqa, osa, oqb, osb), "staged %dx%dx%d" % (M, N, K))


def test_tiny_dense_workload(dev):
    d = wl.tiny_dense()
    (qa, sa, qb, sb), (oqa, osa, oqb, osb) = _quantize_both(d.a, d.b, dev)
    c = fq.fp8_gemm_blockscaled(qa, sa, qb, sb)
    _finish(dev)
    assert_gemm_close(bf16_bits_of(c), oracle.gemm_blockscaled(oqa, osa, oqb, osb), "tiny_dense")


@pytest.mark.parametrize("name", ["dense_fprop", "long_k"])
def test_dense_workloads_sampled(dev, name):
    d = wl.CONFIGS[name]()
    (qa, sa, qb, sb), (oqa, osa, oqb, osb) = _quantize_both(d.a, d.b, dev)
    c = fq.fp8_gemm_blockscaled(qa, sa, qb, sb)
    _finish(dev)
    rows = wl.quad_rows(np.random.default_rng(77), d.M)
    ref = oracle.gemm_blockscaled(oqa, osa, oqb, osb, rows=rows)
    assert_gemm_close(bf16_bits_of(c)[rows], ref, name)


@pytest.mark.parametrize("M,N,K", [
    (1024, 9472, 512),   # 296 wide (128 x 256) tiles: one scale group per tile, the ring's slot moves every tile
    (2048, 4608, 2048),  # 288 wide tiles, four scale groups per tile
    (1024, 4992, 512),   # N/128 odd: 312 128 x 128 tiles on the staged-scale path
    (1000, 4864, 1664),  # 304 128 x 128 tiles, ragged M; K % 512 != 0: scales loaded from global memory
])
def test_dense_many_tiles_full(dev, M, N, K):
    """About two or more tiles per SM, every element compared: each CTA's
    second and later tiles, in every epilogue warp, for both tile widths."""
    rng = np.random.default_rng(M + 5 * N + 11 * K)
    a = rng.standard_normal((M, K)).astype(np.float32) * np.exp(rng.standard_normal(K)).astype(np.float32)
    b = (0.02 * rng.standard_normal((N, K))).astype(np.float32)
    (qa, sa, qb, sb), (oqa, osa, oqb, osb) = _quantize_both(wl.bf16_bits(a), wl.bf16_bits(b), dev)
    c = fq.fp8_gemm_blockscaled(qa, sa, qb, sb)
    _finish(dev)
    ref = oracle.gemm_blockscaled(oqa, osa, oqb, osb)
    assert_gemm_close(bf16_bits_of(c), ref, "dense %dx%dx%d" % (M, N, K))


def test_all_ones_closed_form(dev):
    M, N, K = 256, 512, 1024
    a = torch.ones((M, K), dtype=torch.bfloat16, device=dev)
    b = torch.ones((N, K), dtype=torch.bfloat16, device=dev)
    qa, sa = fq.fp8_quant_act_1x128(a)
    qb, sb = fq.fp8_quant_w_128x128(b)
    c = fq.fp8_gemm_blockscaled(qa, sa, qb, sb)
    _finish(dev)
    s = float(np.float32(1.0) / np.float32(448.0))
    closed = K * (448.0 * s) ** 2
    assert_gemm_close(bf16_bits_of(c), np.full((M, N), closed), "all-ones")


def test_output_rows_beyond_m_untouched(dev):
    """A ragged M writes exactly M rows of the caller's buffer."""
    M, N, K = 130, 256, 256
    rng = np.random.default_rng(5)
    a = wl.bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    b = wl.bf16_bits(rng.standard_normal((N, K)).astype(np.float32))
    (qa, sa, qb, sb), _ = _quantize_both(a, b, dev)
    buf = torch.full((M + 126, N), 7.0, dtype=torch.bfloat16, device=dev)
    fq.fp8_gemm_blockscaled(qa, sa, qb, sb, out=buf[:M])
    _finish(dev)
    assert torch.all(buf[M:] == 7.0)


# ------------------------------------------------------------------ contiguous
def _contiguous_case(dev, d, all_rows=False):
    (qa, sa, qb, sb), (oqa, osa, oqb, osb) = _quantize_both(d.a, d.b, dev)
    mi = torch.from_numpy(d.m_indices).to(dev)
    c = fq.fp8_grouped_gemm_contiguous(qa, sa, qb.view(d.b.shape), sb, mi)
    _finish(dev)
    rows = np.arange(d.M_tot) if all_rows else wl.quad_rows(np.random.default_rng(3), d.M_tot)
    ref = oracle.grouped_contiguous(oqa, osa, oqb, osb, d.m_indices, rows=rows)
    assert_gemm_close(bf16_bits_of(c)[rows], ref, d.name)


def test_contiguous_small(dev):
    _contiguous_case(dev, wl.moe_contiguous(tokens=96, topk=4, E=6, N=384, K=512, seed=21), all_rows=True)


@pytest.mark.parametrize("N,K,tile_n", [(5120, 512, 256), (5120, 2048, 256), (2432, 512, 128)])
def test_contiguous_many_tiles_full(dev, N, K, tile_n):
    """Over 2 x 148 tiles of mixed experts, every element compared; 128 x 256
    tiles when N is a multiple of 256 (staged scales), else 128 x 128."""
    d = wl.moe_contiguous(tokens=512, topk=6, E=8, N=N, K=K, seed=40 + K + N)
    assert (d.M_tot // TILE) * (d.N // tile_n) > 2 * 148
    _contiguous_case(dev, d, all_rows=True)


def test_contiguous_full(dev):
    _contiguous_case(dev, wl.moe_contiguous())


def test_contiguous_skips_out_of_range_blocks(dev):
    d = wl.moe_contiguous(tokens=64, topk=4, E=4, N=256, K=256, seed=8)
    (qa, sa, qb, sb), (oqa, osa, oqb, osb) = _quantize_both(d.a, d.b, dev)
    mi = d.m_indices.copy()
    mi[0] = -1
    mi[-1] = d.E  # out of range too
    out = torch.full((d.M_tot, d.N), 3.0, dtype=torch.bfloat16, device=dev)
    fq.fp8_grouped_gemm_contiguous(qa, sa, qb.view(d.b.shape), sb, torch.from_numpy(mi).to(dev), out=out)
    _finish(dev)
    got = bf16_bits_of(out)
    assert np.all(got[:TILE] == 0x4040) and np.all(got[-TILE:] == 0x4040)  # bf16 3.0 untouched
    ref = oracle.grouped_contiguous(oqa, osa, oqb, osb, mi)
    assert_gemm_close(got[TILE:-TILE], ref[TILE:-TILE], "contiguous middle")


# ------------------------------------------------------------------ masked
def _masked_case(dev, a, b, masked_m, sampled=False):
    E, cap, K = a.shape
    N = b.shape[1]
    (qa, sa, qb, sb), (oqa, osa, oqb, osb) = _quantize_both(a, b, dev)
    qa = qa.view(E, cap, K)
    sa = sa.view(E, cap, K // TILE)
    mm = torch.from_numpy(np.asarray(masked_m, dtype=np.int32)).to(dev)
    out = torch.full((E, cap, N), -5.0, dtype=torch.bfloat16, device=dev)
    fq.fp8_grouped_gemm_masked(qa, sa, qb.view(b.shape), sb, mm, expected_m=int(np.mean(masked_m)), out=out)
    _finish(dev)
    got = bf16_bits_of(out).reshape(E * cap, N)
    oqa3 = oqa.reshape(E, cap, K)
    osa3 = osa.reshape(E, cap, K // TILE)
    valid = np.concatenate([np.arange(e * cap, e * cap + min(cap, max(0, int(masked_m[e])))) for e in range(E)]
                           + [np.zeros(0, np.int64)])
    invalid = np.setdiff1d(np.arange(E * cap), valid)
    assert np.all(got[invalid] == 0xC0A0), "rows at or past masked_m must stay untouched"  # bf16 -5.0
    if not sampled:
        rows = valid
    else:
        # every 32-row quad of every valid tile of every expert
        rng = np.random.default_rng(11)
        rows = []
        for e in range(E):
            m = min(cap, max(0, int(masked_m[e])))
            if m:
                rows.extend(e * cap + wl.quad_rows(rng, m))
        rows = np.asarray(rows, dtype=np.int64)
    if rows.size:
        ref = oracle.grouped_masked(oqa3, osa3, oqb, osb, np.asarray(masked_m, np.int32), rows=rows)
        assert_gemm_close(got[rows], ref, "masked")


def test_masked_small_edge_counts(dev):
    rng = np.random.default_rng(31)
    E, cap, N, K = 6, 256, 384, 512
    a = wl.bf16_bits(rng.standard_normal((E, cap, K)).astype(np.float32))
    b = wl.bf16_bits((0.02 * rng.standard_normal((E, N, K))).astype(np.float32))
    _masked_case(dev, a, b, [0, 1, 128, 129, 256, 255])


def test_masked_all_empty(dev):
    rng = np.random.default_rng(32)
    a = wl.bf16_bits(rng.standard_normal((3, 128, 256)).astype(np.float32))
    b = wl.bf16_bits(rng.standard_normal((3, 256, 256)).astype(np.float32))
    _masked_case(dev, a, b, [0, 0, 0])


def test_masked_out_of_range_counts_clamped(dev):
    rng = np.random.default_rng(33)
    a = wl.bf16_bits(rng.standard_normal((3, 128, 256)).astype(np.float32))
    b = wl.bf16_bits(rng.standard_normal((3, 256, 256)).astype(np.float32))
    _masked_case(dev, a, b, [-4, 500, 77])


@pytest.mark.parametrize("N,tile_n", [(5120, 256), (2432, 128)])
def test_masked_many_tiles_full(dev, N, tile_n):
    """Over 2 x 148 tiles (counts spanning 0..cap), every valid element
    compared and every other row checked untouched; both tile widths."""
    rng = np.random.default_rng(34 + N)
    E, cap, K = 12, 256, 1024
    masked_m = rng.integers(0, cap, size=E, endpoint=True)
    masked_m[:3] = [cap, 129, 0]
    tiles = sum((int(m) + TILE - 1) // TILE for m in masked_m) * (N // tile_n)
    assert tiles > 2 * 148
    a = wl.bf16_bits(rng.standard_normal((E, cap, K)).astype(np.float32))
    b = wl.bf16_bits((0.02 * rng.standard_normal((E, N, K))).astype(np.float32))
    _masked_case(dev, a, b, masked_m)


def test_masked_full_both_gemms(dev):
    d = wl.moe_masked()
    _masked_case(dev, d.a, d.b, d.masked_m, sampled=True)
    _masked_case(dev, d.a2, d.b2, d.masked_m, sampled=True)
