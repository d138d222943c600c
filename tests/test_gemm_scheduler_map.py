"""Host replay of the GEMM's persistent tile scheduler and epilogue ownership.

The GEMM kernel (fp8q_gemm.cuh) walks tiles t = blockIdx.x, +gridDim.x, ...
below a total, maps each t to a tile with get_tile (dense, MoE contiguous,
MoE masked), and its eight epilogue warps each own one TMEM lane quarter
(32 rows) and one half of the tile's columns, storing only rows below the
tile's valid count and columns below N.  For the masked form one warp first
builds the per-expert prefix of tile counts with a chunked warp scan.

These tests restate that arithmetic (and the launcher's grid choice in
fp8q_api.cu) on the CPU for many shapes and grid sizes and check:
  * every valid output element is written exactly once and no other element
    is written (masked rows at or past an expert's count, contiguous blocks
    whose expert index is out of range);
  * every row of B and every scale read lies inside its tensor;
  * the warp-scan prefix equals the plain exclusive prefix sum, for any
    expert count up to the 1024 the kernel's shared-memory prefix holds.
"""
import numpy as np
import pytest

BM, SLAB_K = 128, 128
EPI_WARPS = range(4, 12)


def tile_n(N, K, staged=True, kind="masked", m_tiles=1, num_sms=148):
    """The launcher's tile width (fp8q_api.cu, use_wide_tiles): 256 columns on
    the staged-scale path when N is a multiple of 256 and, for the dense and
    contiguous layouts, 2 x 0.95 x (rounds of wide tiles) <= rounds of
    128-column tiles; else 128."""
    if not (staged and (K // SLAB_K) % 4 == 0 and N % 256 == 0):
        return 128
    if kind == "masked":
        return 256
    r_narrow = -(-(m_tiles * (N // 128)) // num_sms)
    r_wide = -(-(m_tiles * (N // 256)) // num_sms)
    return 256 if 19 * r_wide <= 10 * r_narrow else 128


def masked_rows(masked_m, e, cap):
    m = int(masked_m[e])
    return 0 if m < 0 else min(m, cap)


def warp_scan_prefix(masked_m, cap, n_tiles):
    """build_masked_prefix: lane l sums experts [l*chunk, min(E, (l+1)*chunk)),
    inclusive shuffle-up scan over the 32 lanes, then each lane writes its
    running prefix; lane 31 writes the total at index E."""
    E = len(masked_m)
    chunk = (E + 31) // 32
    prefix = np.full(E + 1, -1, dtype=np.int64)
    local = []
    for lane in range(32):
        e0, e1 = lane * chunk, min(E, lane * chunk + chunk)
        local.append(sum(-(-masked_rows(masked_m, e, cap) // BM) * n_tiles for e in range(e0, e1)))
    incl = list(local)
    off = 1
    while off < 32:
        incl = [incl[l] + (incl[l - off] if l >= off else 0) for l in range(32)]
        off <<= 1
    for lane in range(32):
        e0, e1 = lane * chunk, min(E, lane * chunk + chunk)
        run = incl[lane] - local[lane]
        for e in range(e0, e1):
            prefix[e] = run
            run += -(-masked_rows(masked_m, e, cap) // BM) * n_tiles
    prefix[E] = incl[31]
    return prefix


def get_tile(kind, t, *, M, N, E, n_tiles, m_indices=None, masked_m=None, prefix=None, bn=128):
    """Returns (a_row, b_row, n0, e, rows) or None for a skipped tile."""
    if kind == "masked":
        lo, hi = 0, E
        while hi - lo > 1:
            mid = (lo + hi) >> 1
            if prefix[mid] <= t:
                lo = mid
            else:
                hi = mid
        e = lo
        rows_e = masked_rows(masked_m, e, M)
        mt_count = -(-rows_e // BM)
        local = t - prefix[e]
        nt, mt = divmod(local, mt_count)
        n0 = nt * bn
        return e * M + mt * BM, e * N + n0, n0, e, min(BM, rows_e - mt * BM)
    mt, nt = divmod(t, n_tiles)
    a_row, n0 = mt * BM, nt * bn
    if kind == "contiguous":
        e = int(m_indices[mt])
        if e < 0 or e >= E:
            return None
        rows = BM
    else:
        e, rows = 0, min(BM, M - a_row)
    return a_row, e * N + n0, n0, e, rows


def replay(kind, *, M, N, K, E=1, m_indices=None, masked_m=None, num_sms=148, staged=True):
    """Runs the scheduler and the epilogue stores of every CTA; returns the
    per-element write counts of C (shape [a_rows, N])."""
    BN = tile_n(N, K, staged, kind, (M // BM) if kind == "contiguous" else -(-M // BM), num_sms)
    n_tiles = -(-N // BN)
    nnb = N // 128
    assert K >= SLAB_K and K % SLAB_K == 0
    if kind == "masked":
        m_tiles, a_rows = M // BM, E * M
        prefix = warp_scan_prefix(masked_m, M, n_tiles)
        total = int(prefix[E])
        max_tiles = m_tiles * n_tiles * E
    else:
        m_tiles = -(-M // BM)
        a_rows, prefix = M, None
        total = m_tiles * n_tiles
        max_tiles = total
    grid = min(max_tiles, num_sms)
    writes = np.zeros((a_rows, N), dtype=np.int32)
    if grid <= 0:
        return writes
    for bx in range(grid):
        for t in range(bx, total, grid):
            tile = get_tile(kind, t, M=M, N=N, E=E, n_tiles=n_tiles, m_indices=m_indices, masked_m=masked_m,
                            prefix=prefix, bn=BN)
            if tile is None:
                continue
            a_row, b_row, n0, e, rows = tile
            assert 0 < rows <= BM
            assert 0 <= b_row and b_row + BN <= E * N          # the B box stays inside [E*N, K]
            assert 0 <= a_row < a_rows
            for warp in EPI_WARPS:
                quad, half = warp & 3, (warp - 4) >> 2
                col0 = n0 + half * (BN // 2)
                col_ok = col0 < N
                sb_row = e * nnb + (col0 // 128 if col_ok else 0)
                assert 0 <= sb_row < E * nnb                    # sb is [E*N/128, nkb]
                if staged and (K // SLAB_K) % 4 == 0:
                    # the staged box: BN/128 block rows from the tile's first; this half reads row (half*BN/2)//128
                    box0, box_rows = e * nnb + n0 // 128, max(1, BN // 128)
                    assert (half * (BN // 2)) // 128 < box_rows
                    if col_ok:
                        assert box0 + (half * (BN // 2)) // 128 == sb_row
                    if BN > 128:
                        assert box0 + box_rows <= E * nnb       # a wide tile's box stays inside sb
                for lane in range(32):
                    r = quad * 32 + lane
                    row_ok = r < rows
                    sa_row = a_row + (r if row_ok else 0)
                    assert 0 <= sa_row < a_rows                 # sa is [a_rows, nkb]
                    if row_ok and col_ok:
                        writes[a_row + r, col0:col0 + BN // 2] += 1
    return writes


@pytest.mark.parametrize("M,N,sms", [(1, 128, 148), (128, 256, 148), (300, 384, 5), (4096, 7168, 148),
                                     (129, 128, 1), (1000, 1024, 7)])
@pytest.mark.parametrize("K", [256, 512])
def test_dense_writes_every_element_once(M, N, sms, K):
    """K = 512 takes the staged-scale path, so N % 256 == 0 shapes use wide tiles."""
    w = replay("dense", M=M, N=N, K=K, num_sms=sms)
    assert np.all(w == 1)


def test_tile_width_choice():
    # only whole 256-column blocks on the staged-scale path
    assert tile_n(7168, 7168) == 256 and tile_n(4096, 2048) == 256
    assert tile_n(384, 512) == 128 and tile_n(7168, 1664) == 128 and tile_n(7168, 512, staged=False) == 128
    # dense 4096 x 7168: 896 wide tiles take 7 rounds against 13 of 1792 narrow ones (13.3 > 13): narrow
    assert tile_n(7168, 7168, kind="dense", m_tiles=32) == 128
    # 8192 x 4096: 7 rounds against 14: wide; 2048 x 2048: 1 against 2: wide
    assert tile_n(4096, 7168, kind="dense", m_tiles=64) == 256
    assert tile_n(2048, 16384, kind="dense", m_tiles=16) == 256
    # the MoE contiguous workload (274 row blocks, N = 4096): 30 rounds against 60: wide
    assert tile_n(4096, 7168, kind="contiguous", m_tiles=274) == 256


def test_contiguous_skips_padding_blocks():
    rng = np.random.default_rng(5)
    E, N, blocks = 6, 256, 40
    m_indices = rng.integers(0, E, size=blocks).astype(np.int32)
    m_indices[[3, 17, 39]] = -1          # padding blocks
    m_indices[20] = E                    # out of range: skipped as well
    for sms in (148, 9, 1):
        for K in (128, 512):
            w = replay("contiguous", M=blocks * BM, N=N, K=K, E=E, m_indices=m_indices, num_sms=sms)
            for b in range(blocks):
                want = 1 if 0 <= m_indices[b] < E else 0
                assert np.all(w[b * BM:(b + 1) * BM] == want), (sms, b, K)
        w = replay("contiguous", M=blocks * BM, N=N, K=128, E=E, m_indices=m_indices, num_sms=sms)
        for b in range(blocks):
            want = 1 if 0 <= m_indices[b] < E else 0
            assert np.all(w[b * BM:(b + 1) * BM] == want), (sms, b)


@pytest.mark.parametrize("counts,cap,sms", [
    ([0, 5, 128, 129, 300, 256], 384, 148),
    ([0, 0, 0], 128, 148),               # nothing to do
    ([-3, 1000, 7], 256, 4),             # negative and over-capacity counts are clamped
    ([1] * 70, 128, 148),                # many experts, one ragged row each
    ([127, 0, 0, 0, 129], 256, 3),
])
def test_masked_writes_exactly_the_valid_rows(counts, cap, sms):
    masked_m = np.array(counts, dtype=np.int32)
    E, N = len(counts), 256
    w = replay("masked", M=cap, N=N, K=512, E=E, masked_m=masked_m, num_sms=sms).reshape(E, cap, N)
    for e in range(E):
        valid = masked_rows(masked_m, e, cap)
        assert np.all(w[e, :valid] == 1), e
        assert np.all(w[e, valid:] == 0), e


@pytest.mark.parametrize("E", [1, 2, 31, 32, 33, 100, 257, 1024])
def test_warp_scan_prefix_is_the_exclusive_sum(E):
    rng = np.random.default_rng(E)
    cap, n_tiles = 512, 3
    masked_m = rng.integers(-10, cap + 50, size=E).astype(np.int32)
    masked_m[rng.random(E) < 0.3] = 0
    got = warp_scan_prefix(masked_m, cap, n_tiles)
    per = np.array([-(-masked_rows(masked_m, e, cap) // BM) * n_tiles for e in range(E)], dtype=np.int64)
    want = np.concatenate([[0], np.cumsum(per)])
    assert np.array_equal(got, want)


def test_masked_binary_search_lands_on_nonempty_experts():
    """Experts with no tiles share their prefix with the next one; the search
    for the largest e with prefix[e] <= t must pick the expert that owns t."""
    masked_m = np.array([0, 0, 200, 0, 0, 1, 0], dtype=np.int32)
    cap, N = 256, 128
    prefix = warp_scan_prefix(masked_m, cap, 1)
    owners = [get_tile("masked", t, M=cap, N=N, E=7, n_tiles=1, masked_m=masked_m, prefix=prefix)[3]
              for t in range(int(prefix[-1]))]
    assert owners == [2, 2, 5]
