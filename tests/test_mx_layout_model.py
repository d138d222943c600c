"""Host replay of the E8M0 scale-atom converters (CPU only).

The block-scaled GEMM reads, per 128-row tile and 128-deep slab, a 512-byte
atom whose byte 16*m0 + 4*m1 + j is the E8M0 scale of tile row 32*m1 + m0
for K block j (mx_scales_act_kernel / mx_scales_w_kernel in
fp8q_gemm_mx.cuh).  These tests restate the converters' index arithmetic and
check that every atom byte is written once with the right row's code, and
that the E8M0 code of a power-of-two binary32 scale is its exponent field.
"""
import struct

import numpy as np
import pytest


def e8m0_of(s: float) -> int:
    return (struct.unpack("<I", struct.pack("<f", s))[0] >> 23) & 0xFF


def test_e8m0_code_of_every_power_of_two():
    for e in range(-127, 128):
        s = np.float32(2.0 ** e)   # 2^-127 is a binary32 subnormal
        assert e8m0_of(float(s)) == e + 127


def act_atoms(codes, M, nkb):
    """mx_scales_act_kernel: thread i -> (atom = i >> 5, m0 = i & 31) writes
    16 bytes at atom*512 + 16*m0: rows 32*m1 + m0 (m1 = 0..3), each byte x4."""
    mt_n = -(-M // 128)
    total = mt_n * nkb * 32
    out = np.full(mt_n * nkb * 512, -1, dtype=np.int32)
    for i in range(total):
        m0, atom = i & 31, i >> 5
        mt, kb = divmod(atom, nkb)
        for m1 in range(4):
            row = mt * 128 + 32 * m1 + m0
            b = codes[row, kb] if row < M else 127
            off = atom * 512 + m0 * 16 + m1 * 4
            assert np.all(out[off:off + 4] == -1)
            out[off:off + 4] = b
    return out.reshape(mt_n, nkb, 512)


@pytest.mark.parametrize("M,nkb", [(128, 1), (300, 3), (1, 2)])
def test_activation_atoms(M, nkb):
    rng = np.random.default_rng(M + nkb)
    codes = rng.integers(0, 255, size=(M, nkb))
    atoms = act_atoms(codes, M, nkb)
    assert np.all(atoms >= 0)
    for mt in range(atoms.shape[0]):
        for kb in range(nkb):
            for m in range(128):
                row = mt * 128 + m
                want = codes[row, kb] if row < M else 127
                m0, m1 = m % 32, m // 32
                for j in range(4):
                    assert atoms[mt, kb, 16 * m0 + 4 * m1 + j] == want


def test_weight_atoms():
    """mx_scales_w_kernel: thread i writes bytes 16i .. 16i+15, all the code
    of scale i >> 5 (= nb * nkb + kb)."""
    nb, nkb = 3, 5
    codes = np.arange(nb * nkb) + 100
    out = np.full(nb * nkb * 512, -1)
    for i in range(nb * nkb * 32):
        assert np.all(out[16 * i:16 * i + 16] == -1)
        out[16 * i:16 * i + 16] = codes[i >> 5]
    atoms = out.reshape(nb, nkb, 512)
    for n in range(nb):
        for k in range(nkb):
            assert np.all(atoms[n, k] == codes[n * nkb + k])
