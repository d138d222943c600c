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
    """quant_act_128x1_kernel: one 128x128 block per CTA step; thread t owns
    channels 8*(t%16)..+7 of rows 8*(t/16)..+7; rows past M are skipped."""
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
    """transpose_w_128x128_kernel: block b -> (g, nb, kb); 1024 16-byte chunks
    per block, 4 per thread; output element (g, k, n) written once."""
    nkb, nnb = K // TILE, N // TILE
    blocks = G * nnb * nkb
    out = np.zeros((G, K, N), dtype=np.int32)
    src = np.zeros((G, N, K), dtype=np.int32)
    st = np.zeros((G, nkb, nnb), dtype=np.int32)
    for bx in range(grid):
        b = bx
        while b < blocks:
            g, rem = b // (nnb * nkb), b % (nnb * nkb)
            nb, kb = rem // nkb, rem % nkb
            for t in range(256):
                for i in range(4):
                    c = t + 256 * i
                    row, ch = c >> 3, c & 7
                    src[g, nb * 128 + row, kb * 128 + ch * 16: kb * 128 + ch * 16 + 16] += 1
                    orow = row  # the store loop uses the same chunk numbering on the output side
                    out[g, kb * 128 + orow, nb * 128 + ch * 16: nb * 128 + ch * 16 + 16] += 1
            st[g, kb, nb] += 1
            b += grid
    return src, out, st


@pytest.mark.parametrize("G,N,K,grid", [(1, 128, 128, 1), (1, 256, 384, 2), (3, 128, 256, 5)])
def test_transpose_reads_and_writes_every_element_once(G, N, K, grid):
    src, out, st = transpose_map(G, N, K, grid)
    assert np.all(src == 1) and np.all(out == 1) and np.all(st == 1)


def test_launch_caps_leave_no_work_behind():
    """The launchers cap the grid (SMs x 10, x 16, x 64); the grid-stride loops
    above cover any count of blocks with any positive grid."""
    for blocks, cap in [(10, 1480), (5000, 1480), (1, 2368), (9999, 2368)]:
        grid = min(blocks, cap)
        covered = sum(len(range(bx, blocks, grid)) for bx in range(grid))
        assert covered == blocks
