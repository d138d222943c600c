"""Host replay of the quantizer and transpose kernels' index maps.

Each kernel decides from (block, thread, loop step) which elements it reads
and writes.  These tests replay that arithmetic on the CPU for many shapes
and grid sizes (ragged edges, grids smaller and larger than the work) and
check that every output element is written exactly once, every read stays
inside its tensor, and every scale is written once.  The formulas restate the
kernels' index expressions (fp8q_quant.cuh) and the grid caps of their
launchers (fp8q_api.cu).
"""
import numpy as np
import pytest

TILE = 128


def act_1x128_map(M, K, grid, unroll=2, threads=256):
    """quant_act_1x128_kernel: 8 lanes per tile, `unroll` tiles per lane group
    and iteration, grid-stride over lane groups."""
    tiles = M * (K // TILE)
    ngrp = grid * threads // 8
    written = np.zeros(tiles * 128, dtype=np.int32)   # code bytes
    scales = np.zeros(tiles, dtype=np.int32)
    for grp in range(ngrp):
        t0 = grp
        while t0 - grp < tiles:
            for u in range(unroll):
                t = t0 + u * ngrp
                if t < tiles:
                    for sub in range(8):
                        lo = t * 128 + sub * 16
                        assert t * 256 + sub * 32 + 32 <= tiles * 256  # the 32-byte read
                        written[lo:lo + 16] += 1
                    scales[t] += 1
            t0 += ngrp * unroll
    return written, scales


@pytest.mark.parametrize("M,K,grid", [(1, 128, 1), (3, 384, 2), (257, 640, 7), (4096, 7168, 1480), (64, 128, 1480)])
def test_act_1x128_covers_every_element_once(M, K, grid):
    written, scales = act_1x128_map(M, K, grid)
    assert np.all(written == 1) and np.all(scales == 1)


def act_128x1_map(M, K, grid):
    """quant_act_128x1_kernel<false>: one 128x128 block per CTA step; thread t
    owns channels 8*(t%16)..+7 of rows 8*(t/16)..+7; rows past M are skipped."""
    nkc, nmb = K // TILE, -(-M // TILE)
    blocks = nmb * nkc
    written = np.zeros((M, K), dtype=np.int32)
    scales = np.zeros((nmb, K), dtype=np.int32)
    for bx in range(grid):
        b = bx
        while b < blocks:
            mb, kc = b // nkc, b % nkc
            for t in range(256):
                cg, rg = t & 15, t >> 4
                col0, row0 = kc * 128 + cg * 8, mb * 128 + rg * 8
                assert col0 + 8 <= K
                for r in range(8):
                    row = row0 + r
                    if row < M:
                        written[row, col0:col0 + 8] += 1
                if rg == 0:
                    scales[mb, col0:col0 + 8] += 1
            b += grid
    return written, scales


@pytest.mark.parametrize("M,K,grid", [(1, 128, 1), (200, 256, 3), (1000, 640, 16), (256, 384, 100)])
def test_act_128x1_covers_every_element_once(M, K, grid):
    written, scales = act_128x1_map(M, K, grid)
    assert np.all(written == 1) and np.all(scales == 1)


def transpose_map(G, N, K, grid):
    """transpose_w_128x128_kernel: block b -> (g, nb, kb).  Thread t reads the
    16-byte chunk t % 8 of block rows t / 8 + 32 i (i < 4) and writes its two
    8-byte slots 2c, 2c + 1 to the shared tile at slot s ^ (R / 8) of row R;
    then thread (l = t % 16, j = t / 16) reads slot j ^ l of rows 8l + r
    (r < 8), i.e. the 8x8 bytes at rows 8l.., columns 8j.., and writes them
    transposed at output rows 8j.., columns 8l..  Returns the read and write
    counts and the output as tags of the source elements."""
    nkb, nnb = K // TILE, N // TILE
    blocks = G * nnb * nkb
    out = np.full((G, K, N), -1, dtype=np.int64)
    src = np.zeros((G, N, K), dtype=np.int32)
    writes = np.zeros((G, K, N), dtype=np.int32)
    st = np.zeros((G, nkb, nnb), dtype=np.int32)
    tags = np.arange(G * N * K, dtype=np.int64).reshape(G, N, K)
    for bx in range(grid):
        b = bx
        while b < blocks:
            g, rem = b // (nnb * nkb), b % (nnb * nkb)
            nb, kb = rem // nkb, rem % nkb
            tile = np.full((128, 16, 8), -1, dtype=np.int64)   # [row][physical 8-byte slot][byte]
            tile_writes = np.zeros((128, 16), dtype=np.int32)
            for t in range(256):
                for i in range(4):
                    row, c = (t >> 3) + 32 * i, t & 7
                    r0, c0 = nb * 128 + row, kb * 128 + 16 * c
                    src[g, r0, c0:c0 + 16] += 1
                    x = (row >> 3) & 15
                    for h in range(2):
                        slot = (2 * c + h) ^ x
                        tile[row, slot] = tags[g, r0, c0 + 8 * h:c0 + 8 * h + 8]
                        tile_writes[row, slot] += 1
            assert np.all(tile_writes == 1)            # the swizzle is a permutation of each row's slots
            for t in range(256):
                l, j = t & 15, t >> 4
                block = np.stack([tile[8 * l + r, j ^ l] for r in range(8)])   # [r][c]
                o0, oc = kb * 128 + 8 * j, nb * 128 + 8 * l
                out[g, o0:o0 + 8, oc:oc + 8] = block.T       # lo[c], hi[c] after the register transpose
                writes[g, o0:o0 + 8, oc:oc + 8] += 1
            st[g, kb, nb] += 1
            b += grid
    return src, writes, st, out, tags


def test_transpose_tile_reads_are_conflict_free():
    """Each half-warp's eight-byte shared loads (fixed j, l = 0..15, fixed r)
    cover all 32 banks once: one wavefront per half warp."""
    for r in range(8):
        for j in range(16):
            banks = set()
            for l in range(16):
                addr = (8 * l + r) * 128 + ((j ^ l) << 3)
                banks.update({(addr // 4) % 32, (addr // 4 + 1) % 32})
            assert len(banks) == 32


@pytest.mark.parametrize("G,N,K,grid", [(1, 128, 128, 1), (1, 256, 384, 2), (3, 128, 256, 5)])
def test_transpose_reads_and_writes_every_element_once(G, N, K, grid):
    src, writes, st, out, tags = transpose_map(G, N, K, grid)
    assert np.all(src == 1) and np.all(writes == 1) and np.all(st == 1)
    assert np.array_equal(out, np.swapaxes(tags, 1, 2))


def test_transpose_warp_stores_are_full_rows():
    """Per store instruction (fixed c) a warp's lanes write 8 bytes each at
    output columns 8l of rows 8j + c: two rows, 128 contiguous bytes each."""
    for w in range(8):
        for c in range(8):
            rows = {}
            for t in range(32 * w, 32 * w + 32):
                l, j = t & 15, t >> 4
                rows.setdefault(8 * j + c, []).append(8 * l)
            assert len(rows) == 2 and all(sorted(v) == list(range(0, 128, 8)) for v in rows.values())


def test_launch_caps_leave_no_work_behind():
    """The launchers cap the grid (SMs x 2, x 10, x 16, x 64); the grid-stride
    loops above cover any count of blocks with any positive grid."""
    for blocks, cap in [(10, 1480), (5000, 1480), (1, 2368), (9999, 2368), (1792, 296), (5, 296)]:
        grid = min(blocks, cap)
        covered = sum(len(range(bx, blocks, grid)) for bx in range(grid))
        assert covered == blocks


# ---------------------------------------------------------------- token-contiguous codes
def byte_perm(x, y, s):
    """__byte_perm: result byte i is byte (s >> 4i) & 7 of the 8 bytes {x, y} (x low)."""
    src = [(x >> (8 * i)) & 0xFF for i in range(4)] + [(y >> (8 * i)) & 0xFF for i in range(4)]
    return sum(src[(s >> (4 * i)) & 7] << (8 * i) for i in range(4))


def transpose4x4_bytes(w):
    x0, x2 = byte_perm(w[0], w[2], 0x5410), byte_perm(w[0], w[2], 0x7632)
    x1, x3 = byte_perm(w[1], w[3], 0x5410), byte_perm(w[1], w[3], 0x7632)
    return [byte_perm(x0, x1, 0x6240), byte_perm(x0, x1, 0x7351), byte_perm(x2, x3, 0x6240),
            byte_perm(x2, x3, 0x7351)]


def transpose8x8_bytes(lo, hi):
    lo, hi = list(lo), list(hi)
    lo[0:4] = transpose4x4_bytes(lo[0:4])
    lo[4:8] = transpose4x4_bytes(lo[4:8])
    hi[0:4] = transpose4x4_bytes(hi[0:4])
    hi[4:8] = transpose4x4_bytes(hi[4:8])
    for i in range(4):
        hi[i], lo[4 + i] = lo[4 + i], hi[i]
    return lo, hi


def test_byte_transpose_8x8():
    rng = np.random.default_rng(0)
    for _ in range(50):
        m = rng.integers(0, 256, size=(8, 8), dtype=np.uint8)
        words = m.view("<u4").reshape(8, 2)
        lo, hi = transpose8x8_bytes([int(v) for v in words[:, 0]], [int(v) for v in words[:, 1]])
        got = np.array([[lo[c], hi[c]] for c in range(8)], dtype="<u4").view(np.uint8).reshape(8, 8)
        assert np.array_equal(got, m.T)


def act_128x1_t_map(M, K, grid, Mp=None):
    """quant_act_128x1_kernel<true>: per 128x128 block, thread (cg = t % 16,
    rg = t / 16) writes channel rows cg*8+c of the shared tile (the block's
    spent stage) at physical 8-byte slot rg ^ cg; the store loop reads row c >> 3, 16-byte chunk
    (c & 7) ^ (row >> 4), swapping halves when (row >> 3) is odd, and writes
    qt[kc*128 + row, mb*128 + 16*(c & 7) ...].  Returns the transposed codes
    of a matrix of distinct token/channel tags and the write counts."""
    Mp = Mp or -(-M // 128) * 128
    nkc = K // 128
    blocks = (Mp // 128) * nkc
    # tag of x[m, k] = (m, k) packed; the "code" of a token past M is 0
    out = np.full((K, Mp), -1, dtype=np.int64)
    writes = np.zeros((K, Mp), dtype=np.int32)
    for bx in range(grid):
        for b in range(bx, blocks, grid):
            mb, kc = divmod(b, nkc)
            tile = np.full((128, 16), -1, dtype=object)   # [channel row][physical 8-byte slot] -> 8 token tags
            for t in range(256):
                cg, rg = t & 15, t >> 4
                for c in range(8):
                    row = cg * 8 + c
                    toks = []
                    for r in range(8):
                        m, k = mb * 128 + rg * 8 + r, kc * 128 + cg * 8 + c
                        toks.append(m * K + k + 1 if m < M else 0)
                    slot = rg ^ cg
                    assert tile[row, slot] == -1
                    tile[row, slot] = toks
            for t in range(256):
                for i in range(4):
                    c = t + 256 * i
                    row, ch = c >> 3, c & 7
                    swz = row >> 3
                    p = ch ^ (swz >> 1)
                    halves = [tile[row, 2 * p], tile[row, 2 * p + 1]]
                    if swz & 1:
                        halves = halves[::-1]
                    vals = halves[0] + halves[1]
                    orow, ocol = kc * 128 + row, mb * 128 + ch * 16
                    out[orow, ocol:ocol + 16] = vals
                    writes[orow, ocol:ocol + 16] += 1
    return out, writes


@pytest.mark.parametrize("M,K,grid,Mp", [(128, 128, 1, 128), (200, 256, 3, 256), (300, 128, 2, 512),
                                         (0, 128, 1, 512)])
def test_act_128x1_t_writes_the_transpose(M, K, grid, Mp):
    out, writes = act_128x1_t_map(M, K, grid, Mp)
    assert np.all(writes == 1)
    m = np.arange(Mp)[None, :]
    k = np.arange(K)[:, None]
    want = np.where(m < M, m * K + k + 1, 0)
    assert np.array_equal(out, want)


def test_act_128x1_t_shared_store_conflicts():
    """Per warp store (fixed c), the 32 lanes' 8-byte slots cover every
    8-byte bank slot of the 128-byte rows exactly twice: two wavefronts."""
    for w in range(8):
        for c in range(8):
            slots = [(((t & 15) * 8 + c) * 128 + (((t >> 4) ^ (t & 15)) << 3)) % 128 // 8
                     for t in range(32 * w, 32 * w + 32)]
            assert sorted(slots) == sorted(list(range(16)) * 2)


# ---------------------------------------------------------------- token-axis staging
TOK_STAGES = 3
TOK_BLOCK_BYTES = 128 * 256


def token_axis_fetch_chunks():
    """The copy map of one block: 16-byte chunk c = t + 256 i (t < 256,
    i < 8) is token c >> 4, channels 8 (c & 15) .. +7, at shared byte
    (c >> 4) * 256 + (c & 15) * 16 of the stage."""
    for t in range(256):
        for i in range(8):
            c = t + 256 * i
            row, ch = c >> 4, c & 15
            yield t, row, ch, row * 256 + ch * 16


def test_token_axis_copies_fill_each_stage_once_in_bounds():
    seen = np.zeros(TOK_BLOCK_BYTES, dtype=np.int32)
    for _, row, ch, off in token_axis_fetch_chunks():
        assert 0 <= off and off + 16 <= TOK_BLOCK_BYTES
        assert off == row * 256 + ch * 16 and row < 128 and ch < 16
        seen[off:off + 16] += 1
    assert np.all(seen == 1)
    # a warp's copy instruction (fixed i) covers two whole 256-byte token rows
    for w in range(8):
        for i in range(8):
            rows = {(t + 256 * i) >> 4 for t in range(32 * w, 32 * w + 32)}
            assert len(rows) == 2


def test_token_axis_register_reads_match_the_staged_layout():
    """Thread (cg = t % 16, rg = t / 16) reads its 8 tokens x 8 channels at
    stage byte (rg*8 + r) * 256 + cg * 16: the chunk the copy map put there."""
    where = {}
    for _, row, ch, off in token_axis_fetch_chunks():
        where[off] = (row, ch * 8)
    for t in range(256):
        cg, rg = t & 15, t >> 4
        for r in range(8):
            assert where[(rg * 8 + r) * 256 + cg * 16] == (rg * 8 + r, cg * 8)


def test_token_axis_copy_sources_stay_in_bounds():
    """Tokens past M are zero-filled: no byte is read for them; the other
    copies read inside x [M, K]."""
    for M, K in [(1, 128), (200, 256), (129, 384)]:
        nkc, nmb = K // 128, -(-M // 128)
        for b in range(nmb * nkc):
            mb, kc = divmod(b, nkc)
            for _, row, ch, _ in token_axis_fetch_chunks():
                grow = mb * 128 + row
                if grow < M:
                    src = (grow * K + kc * 128 + ch * 8) * 2
                    assert 0 <= src and src + 16 <= M * K * 2


def token_axis_pipeline(blocks, grid):
    """Replays the kernel's stage bookkeeping per CTA: the prologue fills
    stages 0 .. S-2 with the CTA's first blocks; iteration i (block
    blockIdx + i * grid, stage st = i % S) refills the stage of iteration
    i - 1 with block i + S - 1, commits one group (possibly empty) and waits
    until at most S - 1 groups are pending.  Checks that a refill only hits a
    stage whose block every thread has finished with, that the block read is
    the one copied into the stage, and that its copy group is complete."""
    order = []
    for bx in range(min(blocks, grid)):
        stage = [None] * TOK_STAGES        # block held (or being filled) per stage
        groups = []                         # committed groups, in order: block or None
        for j in range(TOK_STAGES - 1):
            bj = bx + j * grid
            if bj < blocks:
                stage[j] = bj
            groups.append(bj if bj < blocks else None)
        st, i, b = 0, 0, bx
        done = set()
        while b < blocks:
            bn = b + (TOK_STAGES - 1) * grid
            refill = TOK_STAGES - 1 if st == 0 else st - 1
            if bn < blocks:
                assert stage[refill] is None or stage[refill] in done
                stage[refill] = bn
            groups.append(bn if bn < blocks else None)
            complete = groups[:len(groups) - (TOK_STAGES - 1)]   # wait_group(S - 1)
            assert b in complete
            assert stage[st] == b
            order.append(b)
            done.add(b)
            b += grid
            i += 1
            st = 0 if st + 1 == TOK_STAGES else st + 1
    return order


@pytest.mark.parametrize("blocks,grid", [(1, 296), (5, 296), (296, 296), (297, 296), (1792, 296), (40, 3),
                                         (7, 2), (3, 1)])
def test_token_axis_pipeline_processes_every_block_once(blocks, grid):
    order = token_axis_pipeline(blocks, grid)
    assert sorted(order) == list(range(blocks))


def test_token_axis_shared_memory_fits_the_ctas_per_sm():
    """Three 32 KB stages plus the 4 KB channel-maxima array per CTA, two CTAs
    per SM, within the 228 KB an SM offers (1 KB reserved per CTA)."""
    per_cta = TOK_STAGES * TOK_BLOCK_BYTES + 8 * 16 * 8 * 4 + 1024
    assert 2 * per_cta <= 228 * 1024
    assert TOK_STAGES * TOK_BLOCK_BYTES <= 227 * 1024


# ---------------------------------------------------------------- per-element exact codes
def nonzero_bytes(d):
    """Restates the quantizers' nonzero_bytes: bit 8j + 7 set when byte j of d is nonzero."""
    return (((d & 0x7F7F7F7F) + 0x7F7F7F7F) | d) & 0x80808080


def test_nonzero_bytes_marks_exactly_the_nonzero_bytes():
    rng = np.random.default_rng(3)
    words = [0, 0xFFFFFFFF, 0x80808080, 0x01010101, 0x7F7F7F7F, 0x00800001]
    words += [int(v) for v in rng.integers(0, 2 ** 32, 2000, dtype=np.uint64)]
    # every byte value in every position, the other bytes zero
    words += [b << (8 * j) for j in range(4) for b in range(256)]
    for d in words:
        want = sum(0x80 << (8 * j) for j in range(4) if (d >> (8 * j)) & 0xFF)
        assert nonzero_bytes(d) == want, hex(d)


def test_code_byte_names_its_source_element():
    """Code word i of a lane's 16 codes holds elements 4i .. 4i+3: byte j is the
    bf16 at word 2i + j/2, half j%2 (low half first), the order in which the
    packed products are converted.  bf16_of_pair must pick that element."""
    bf16 = np.arange(16, dtype=np.uint32) + 0x3F80      # distinct bf16 patterns, element e at index e
    w = [int(bf16[2 * k]) | (int(bf16[2 * k + 1]) << 16) for k in range(8)]
    for i in range(4):
        # conversion order: pairs (w[2i] low, high), (w[2i+1] low, high) -> bytes 0..3
        converted = [w[2 * i] & 0xFFFF, w[2 * i] >> 16, w[2 * i + 1] & 0xFFFF, w[2 * i + 1] >> 16]
        for j in range(4):
            word = w[2 * i + 1] if j & 2 else w[2 * i]
            picked = (word >> 16) if j & 1 else (word & 0xFFFF)
            assert picked == converted[j] == int(bf16[4 * i + j])


def test_token_axis_channel_maxima_reach_their_channel_thread():
    """Thread (cg, lane < 16) stores its packed maxima word i (channels
    8 cg + 2i, low half, and 8 cg + 2i + 1, high half) at col_max[warp][cg][i];
    channel thread t < 128 reads word (t & 7) >> 1 of [warp][t >> 3], half t & 1."""
    stored = {}
    for cg in range(16):
        for i in range(4):
            stored[(cg, i, 0)] = 8 * cg + 2 * i
            stored[(cg, i, 1)] = 8 * cg + 2 * i + 1
    for t in range(128):
        assert stored[(t >> 3, (t & 7) >> 1, t & 1)] == t
