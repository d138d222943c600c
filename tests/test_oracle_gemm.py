"""Pins for the oracle's block-scaled GEMMs and the accumulation model (CPU).

What fixes the answer (the promotion rule of Figure 7 (b) in "The Insider
Secrets Of Deepseek Discovered" makes the promoted product equal the product
of the dequantized inputs):
* a closed form (all-ones inputs);
* inputs whose every group has amax 448, so all scales are 1 and the product
  reduces to a textbook matmul of E4M3 values (PyTorch decode + numpy matmul,
  exact in float64);
* the dequantized-input identity sum_k (sa*qa)(sb*qb) evaluated by numpy's
  matmul with no slab structure, on non-square shapes with random scales (a
  transposed operand, a wrong scale index or a dropped slab fails it);
* grouped layouts reduce to per-expert dense products;
* the limited-precision model on hand-worked cases, and its qualitative
  behaviour (drift grows with K; promotion removes it).
"""
import numpy as np
import pytest
import torch

from workloads import bf16_bits, bf16_to_f32, long_k, moe_contiguous, moe_masked, tiny_dense

TILE = 128


def _decode(q):
    return torch.from_numpy(np.ascontiguousarray(q)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _dequant_act(q, s):
    return _decode(q) * np.repeat(s.astype(np.float64), TILE, axis=-1)


def _dequant_w(q, s):
    return _decode(q) * np.repeat(np.repeat(s.astype(np.float64), TILE, axis=-2), TILE, axis=-1)


def test_all_ones_closed_form(orc):
    M, N, K = 3, 256, 640
    a = np.full((M, K), 0x3F80, dtype=np.uint16)  # bf16 1.0
    b = np.full((N, K), 0x3F80, dtype=np.uint16)
    qa, sa = orc.quant_act_1x128(a)
    qb, sb = orc.quant_w_128x128(b)
    s = float(np.float32(1.0) / np.float32(448.0))
    assert np.all(sa == np.float32(s)) and np.all(sb == np.float32(s))
    assert np.all(qa == 0x7E) and np.all(qb == 0x7E)
    C = orc.gemm_blockscaled(qa, sa, qb, sb)
    closed = K * (448.0 * s) ** 2
    assert np.allclose(C, closed, rtol=1e-15, atol=0)
    assert abs(closed - K) < K * 1e-6  # 448 * fl32(1/448) is within 1e-7 of 1


def test_unit_scales_reduce_to_textbook_matmul(orc):
    rng = np.random.default_rng(21)
    M, N, K = 130, 384, 512
    a = rng.uniform(-400, 400, size=(M, K)).astype(np.float32)
    b = rng.uniform(-400, 400, size=(N, K)).astype(np.float32)
    a[:, ::TILE] = 448.0
    b[::TILE, ::TILE] = -448.0
    qa, sa = orc.quant_act_1x128(bf16_bits(a))
    qb, sb = orc.quant_w_128x128(bf16_bits(b))
    assert np.all(sa == 1.0) and np.all(sb == 1.0)
    C = orc.gemm_blockscaled(qa, sa, qb, sb)
    ref = _decode(qa) @ _decode(qb).T  # every partial sum is exact in float64
    assert np.array_equal(C, ref)


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (77, 256, 384), (130, 384, 1024)])
def test_dequantized_input_identity(orc, M, N, K):
    rng = np.random.default_rng(M * 7 + N + K)
    a = rng.standard_normal((M, K)).astype(np.float32) * np.exp(rng.uniform(-3, 3, size=(1, K))).astype(np.float32)
    b = (0.02 * rng.standard_normal((N, K))).astype(np.float32)
    qa, sa = orc.quant_act_1x128(bf16_bits(a))
    qb, sb = orc.quant_w_128x128(bf16_bits(b))
    C = orc.gemm_blockscaled(qa, sa, qb, sb)
    ref = _dequant_act(qa, sa) @ _dequant_w(qb, sb).T
    scale = np.abs(_dequant_act(qa, sa)) @ np.abs(_dequant_w(qb, sb)).T
    assert np.all(np.abs(C - ref) <= 1e-13 * scale + 1e-300)
    # the slab structure is really there: K = 128 is sa * sb^T times one partial
    if K == 128:
        part = _decode(qa) @ _decode(qb).T
        assert np.allclose(C, sa.astype(np.float64) * np.repeat(sb.astype(np.float64).T, TILE, axis=1) * part,
                           rtol=1e-15, atol=0)


def test_row_subset_matches_full(orc):
    d = tiny_dense(seed=9, M=200)
    qa, sa = orc.quant_act_1x128(d.a)
    qb, sb = orc.quant_w_128x128(d.b)
    full = orc.gemm_blockscaled(qa, sa, qb, sb)
    rows = [0, 5, 127, 128, 199]
    sub = orc.gemm_blockscaled(qa, sa, qb, sb, rows=rows)
    assert np.array_equal(sub, full[rows])


def test_grouped_contiguous_reduces_to_dense(orc):
    d = moe_contiguous(tokens=48, topk=4, E=6, N=256, K=384)
    qa, sa = orc.quant_act_1x128(d.a)
    qb, sb = orc.quant_w_128x128(d.b)
    C = orc.grouped_contiguous(qa, sa, qb, sb, d.m_indices)
    for blk, e in enumerate(d.m_indices):
        r = slice(blk * TILE, (blk + 1) * TILE)
        ref = orc.gemm_blockscaled(np.ascontiguousarray(qa[r]), np.ascontiguousarray(sa[r]),
                                   np.ascontiguousarray(qb[e]), np.ascontiguousarray(sb[e]))
        assert np.array_equal(C[r], ref)
    # pad rows (zero inputs) give zero output
    r0 = 0
    for e in range(d.E):
        c = int(d.counts[e])
        p = (c + TILE - 1) // TILE * TILE
        assert np.all(C[r0 + c:r0 + p] == 0.0)
        r0 += p
    # out-of-range expert index: block left untouched
    mi = d.m_indices.copy()
    mi[0] = -1
    C2 = orc.grouped_contiguous(qa, sa, qb, sb, mi)
    assert np.all(np.isnan(C2[:TILE])) and np.array_equal(C2[TILE:], C[TILE:])


def test_grouped_contiguous_uses_each_blocks_expert(orc):
    """Swapping two experts' weights changes exactly the rows of their blocks."""
    d = moe_contiguous(tokens=64, topk=2, E=4, N=128, K=256, seed=12)
    qa, sa = orc.quant_act_1x128(d.a)
    qb, sb = orc.quant_w_128x128(d.b)
    C = orc.grouped_contiguous(qa, sa, qb, sb, d.m_indices)
    perm = np.array([1, 0, 2, 3])
    C2 = orc.grouped_contiguous(qa, sa, np.ascontiguousarray(qb[perm]), np.ascontiguousarray(sb[perm]),
                                d.m_indices)
    changed = np.any(C2 != C, axis=1).reshape(-1, TILE).any(axis=1)
    touched = np.isin(d.m_indices, [0, 1]) & (np.repeat(d.counts, 1)[d.m_indices] > 0)
    assert np.array_equal(changed, touched)


def test_grouped_masked_reduces_to_dense(orc):
    d = moe_masked(E=5, cap=256, N=256, K=384, second=False, seed=13)
    d.masked_m[:] = [0, 1, 128, 200, 256]
    qa, sa = orc.quant_act_1x128(d.a.reshape(-1, d.a.shape[-1]))
    qa, sa = qa.reshape(d.a.shape), sa.reshape(d.E, d.cap, -1)
    qb, sb = orc.quant_w_128x128(d.b)
    C = orc.grouped_masked(qa, sa, qb, sb, d.masked_m)
    for e in range(d.E):
        m = int(d.masked_m[e])
        ref = orc.gemm_blockscaled(np.ascontiguousarray(qa[e]), np.ascontiguousarray(sa[e]),
                                   np.ascontiguousarray(qb[e]), np.ascontiguousarray(sb[e]))
        assert np.array_equal(C[e, :m], ref[:m])
        assert np.all(np.isnan(C[e, m:])), "rows at or past masked_m stay unwritten"
    rows = [0, 256 + 0, 2 * 256 + 127, 3 * 256 + 199, 3 * 256 + 200, 4 * 256 + 255]
    sub = orc.grouped_masked(qa, sa, qb, sb, d.masked_m, rows=rows)
    flat = C.reshape(-1, C.shape[-1])
    assert np.array_equal(np.isnan(sub), np.isnan(flat[rows]))
    assert np.array_equal(np.nan_to_num(sub), np.nan_to_num(flat[rows]))


# ---------------------------------------------------------------- accumulation model
def _ones_case(K, N=128):
    qa = np.full((1, K), 0x38, dtype=np.uint8)  # 1.0
    qb = np.full((N, K), 0x38, dtype=np.uint8)
    sa = np.ones((1, K // TILE), dtype=np.float32)
    sb = np.ones((N // TILE, K // TILE), dtype=np.float32)
    return qa, sa, qb, sb


@pytest.mark.parametrize("p,group,interval,K,expect", [
    (2, 1, 0, 128, 4.0),      # 1,2,3,4 then 5 -> 4 (two bits kept): stuck at 2^p
    (3, 1, 0, 128, 8.0),
    (2, 1, 128, 256, 8.0),    # restarted every 128: 4 + 4
    (1, 32, 0, 128, 64.0),    # 32, 64, 96 -> 64, 64+32 -> 64
    (2, 32, 0, 128, 128.0),   # 32, 64, 96 (two bits), 128: exact
    (53, 1, 0, 1024, 1024.0),
])
def test_limited_accumulation_hand_cases(orc, p, group, interval, K, expect):
    qa, sa, qb, sb = _ones_case(K)
    C = orc.gemm_limited_acc(qa, sa, qb, sb, p_bits=p, group=group, interval=interval)
    assert np.all(C == expect)


def test_limited_accumulation_full_precision_is_exact(orc):
    d = tiny_dense(seed=2, M=16)
    qa, sa = orc.quant_act_1x128(d.a)
    qb, sb = orc.quant_w_128x128(d.b)
    exact = orc.gemm_blockscaled(qa, sa, qb, sb)
    C = orc.gemm_limited_acc(qa, sa, qb, sb, p_bits=53, group=1, interval=128)
    assert np.allclose(C, exact, rtol=1e-13, atol=1e-13)


def test_limited_accumulation_rejects_mixed_scales_in_interval(orc):
    d = tiny_dense(seed=2, M=4)
    qa, sa = orc.quant_act_1x128(d.a)
    qb, sb = orc.quant_w_128x128(d.b)
    with pytest.raises(ValueError):
        orc.gemm_limited_acc(qa, sa, qb, sb, interval=0)


def _per_tensor(orc, x):
    q, s = orc.quant_tensor(x)
    return q, s


def test_drift_grows_with_k_and_promotion_removes_it(orc):
    """Long-K stress inputs (U[-1,1] + 0.5), per-tensor scales, 14-bit
    accumulator: the unpromoted error grows with K; with promotion every 128
    it stays orders of magnitude smaller."""
    d = long_k(M=4, N=128, K=16384, seed=2)
    rel_unpromoted, rel_promoted = [], []
    for K in (512, 2048, 4096, 16384):
        a = np.ascontiguousarray(d.a[:, :K])
        b = np.ascontiguousarray(d.b[:, :K])
        qa, s_a = _per_tensor(orc, a)
        qb, s_b = _per_tensor(orc, b)
        sa = np.full((a.shape[0], K // TILE), s_a, dtype=np.float32)
        sb = np.full((b.shape[0] // TILE, K // TILE), s_b, dtype=np.float32)
        exact = orc.gemm_blockscaled(qa, sa, qb, sb)
        unp = orc.gemm_limited_acc(qa, sa, qb, sb, p_bits=14, group=32, interval=0)
        pro = orc.gemm_limited_acc(qa, sa, qb, sb, p_bits=14, group=32, interval=128)
        rel_unpromoted.append(np.max(np.abs(unp - exact) / np.abs(exact)))
        rel_promoted.append(np.max(np.abs(pro - exact) / np.abs(exact)))
    assert all(x < y for x, y in zip(rel_unpromoted, rel_unpromoted[1:])), rel_unpromoted
    assert rel_unpromoted[2] > 10 * rel_promoted[2], (rel_unpromoted, rel_promoted)
    assert max(rel_promoted) < 2e-3


# --------------------------------------------------------------------------- backward GEMMs (oracle side)
def _rand_bits(rng, shape, scale=1.0, outliers=0):
    x = (scale * rng.standard_normal(shape)).astype(np.float32)
    if outliers:
        idx = rng.choice(x.size, size=outliers, replace=False)
        x.reshape(-1)[idx] *= 100.0
    return bf16_bits(x)


def test_token_axis_tiles_are_transposed_1x128(orc):
    """128x1 tiles of X are the 1x128 tiles of X^T: same codes, same scales."""
    rng = np.random.default_rng(30)
    x = _rand_bits(rng, (256, 384), outliers=7)
    q, s = orc.quant_act_128x1(x)
    qt, st = orc.quant_act_1x128(np.ascontiguousarray(x.T))
    assert np.array_equal(q, qt.T)
    assert np.array_equal(s.view(np.uint32), st.T.view(np.uint32))


def test_token_axis_ragged_last_group(orc):
    """A ragged last group of tokens takes its scale from its own rows only."""
    x = np.zeros((200, 2), dtype=np.float32)
    x[:128, 0] = 1.0
    x[5, 0] = 448.0          # first group of column 0: amax 448 -> scale 1
    x[128:, 0] = 2.0         # last group (72 rows): amax 2 -> scale fl32(2/448)
    x[150, 1] = -3.5         # column 1: only the last group is non-zero
    q, s = orc.quant_act_128x1(bf16_bits(x))
    assert s.shape == (2, 2)
    assert s[0, 0] == 1.0 and s[0, 1] == 1.0  # zero group -> 1
    assert s[1, 0] == np.float32(np.float32(2.0) / np.float32(448.0))
    assert s[1, 1] == np.float32(np.float32(3.5) / np.float32(448.0))
    assert q[5, 0] == 0x7E and q[0, 0] == orc.e4m3_encode(1.0)
    assert q[150, 1] == 0xFE and np.all(q[128:, 0] == 0x7E)


def test_1d1d_with_blockwise_equal_scales_is_the_blockscaled_gemm(orc):
    rng = np.random.default_rng(31)
    M, N, K = 96, 256, 384
    qa, sa = orc.quant_act_1x128(_rand_bits(rng, (M, K), outliers=3))
    qb, sb = orc.quant_w_128x128(_rand_bits(rng, (N, K), scale=0.02))
    c_block = orc.gemm_blockscaled(qa, sa, qb, sb)
    c_1d1d = orc.gemm_1d1d(qa, sa, qb, np.repeat(sb, TILE, axis=0))
    assert np.array_equal(c_block, c_1d1d)


def test_1d1d_is_the_dequantized_product(orc):
    """Per-row scales on both sides: the result is the product of the
    dequantized operands (a library float64 matmul of decoded codes times
    scales), to float64 rounding."""
    rng = np.random.default_rng(32)
    M, N, K = 64, 160, 512
    qa = rng.integers(0, 256, (M, K), dtype=np.uint8)
    qb = rng.integers(0, 256, (N, K), dtype=np.uint8)
    qa[(qa & 0x7F) == 0x7F] = 0  # no NaN codes
    qb[(qb & 0x7F) == 0x7F] = 0
    sa = rng.uniform(0.5, 2.0, (M, K // TILE)).astype(np.float32)
    sb = rng.uniform(0.5, 2.0, (N, K // TILE)).astype(np.float32)
    deq_a = _decode(qa) * np.repeat(sa.astype(np.float64), TILE, axis=1)
    deq_b = _decode(qb) * np.repeat(sb.astype(np.float64), TILE, axis=1)
    ref = deq_a @ deq_b.T
    got = orc.gemm_1d1d(qa, sa, qb, sb)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_wgrad_and_dgrad_compose_from_the_quantizers(orc):
    """dW = dY^T X on token-axis tiles and dX = dY W on the forward tiles equal
    the products of the dequantized tensors (library matmul)."""
    rng = np.random.default_rng(33)
    M, N, K = 256, 256, 384  # tokens, output channels, input channels
    dy = _rand_bits(rng, (M, N), outliers=5)
    x = _rand_bits(rng, (M, K), outliers=5)
    w = _rand_bits(rng, (N, K), scale=0.02)
    q_dy, s_dy = orc.quant_act_128x1(dy)
    q_x, s_x = orc.quant_act_128x1(x)
    dw = orc.wgrad(q_dy, s_dy, q_x, s_x)
    deq_dy = _decode(q_dy) * np.repeat(s_dy.astype(np.float64), TILE, axis=0)
    deq_x = _decode(q_x) * np.repeat(s_x.astype(np.float64), TILE, axis=0)
    ref_w = deq_dy.T @ deq_x
    assert dw.shape == (N, K)
    assert np.allclose(dw, ref_w, rtol=1e-12, atol=1e-12 * np.abs(ref_w).max())
    q_dy1, s_dy1 = orc.quant_act_1x128(dy)
    q_w, s_w = orc.quant_w_128x128(w)
    dx = orc.dgrad(q_dy1, s_dy1, q_w, s_w)
    ref_x = (_decode(q_dy1) * np.repeat(s_dy1.astype(np.float64), TILE, axis=1)) @ (
        _decode(q_w) * np.repeat(np.repeat(s_w.astype(np.float64), TILE, axis=0), TILE, axis=1))
    assert dx.shape == (M, K)
    assert np.allclose(dx, ref_x, rtol=1e-12, atol=1e-12 * np.abs(ref_x).max())
