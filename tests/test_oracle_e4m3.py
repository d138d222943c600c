"""Pins for the oracle's E4M3 encode/decode (CPU only).

What fixes the answer: the 1-4-3 bit layout ("O que e FP8?" on the DeepGEMM
announcement page; "Unified E4M3" on the codingmall DeepSeek-V3 FP8 page),
hand-computed boundary encodings (tests/golden/e4m3_encodings.txt),
PyTorch's independent float8_e4m3fn conversion, and an exhaustive comparison
with a second, search-based encoder.
"""
import math

import numpy as np
import pytest
import torch

from conftest import golden_lines, hexfloat


def _golden():
    enc, dec = [], []
    for tok in golden_lines("e4m3_encodings.txt"):
        if tok[0] == "decode":
            dec.append((int(tok[1], 16), hexfloat(tok[2])))
        else:
            enc.append((hexfloat(tok[0]), int(tok[1], 16)))
    return enc, dec


def test_golden_encodings(orc):
    enc, _ = _golden()
    assert len(enc) >= 30
    for v, code in enc:
        assert orc.e4m3_encode(v) == code, (v.hex() if math.isfinite(v) else v, hex(code))
        assert orc.e4m3_encode_by_search(v) == code, v


def test_golden_decodings(orc):
    _, dec = _golden()
    for code, v in dec:
        got = orc.e4m3_decode(code)
        if math.isnan(v):
            assert math.isnan(got)
        else:
            assert got == v and math.copysign(1.0, got) == math.copysign(1.0, v), (hex(code), got, v)


def test_decode_all_codes_vs_torch(orc):
    """All 256 codes against PyTorch's float8_e4m3fn -> float32 conversion."""
    table = orc.e4m3_decode_table()
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan_ref = np.isnan(ref)
    assert np.array_equal(np.isnan(table), nan_ref)
    assert nan_ref.sum() == 2  # 0x7F and 0xFF only
    assert np.array_equal(table[~nan_ref], ref[~nan_ref])
    assert np.array_equal(np.signbit(table[~nan_ref]), np.signbit(ref[~nan_ref]))


def test_decode_grid_properties(orc):
    t = orc.e4m3_decode_table()
    pos = t[:127]
    assert np.all(np.diff(pos) > 0), "codes 0x00..0x7E must be strictly increasing"
    assert pos[-1] == 448.0 and pos[1] == 2.0 ** -9 and pos[8] == 2.0 ** -6
    assert np.array_equal(t[128:255], -pos)  # sign bit mirrors
    # every value is an integer multiple of 2^-9 with at most 4 significant bits
    assert np.all(np.mod(pos * 2 ** 9, 1) == 0)


def test_encode_decode_roundtrip(orc):
    for c in list(range(0x7F)) + list(range(0x80, 0xFF)):
        assert orc.e4m3_encode(orc.e4m3_decode(c)) == c, hex(c)


def test_encode_vs_torch_cast_dense_range(orc):
    """Every third binary32 pattern with |v| in [2^-12, 448], both signs,
    against PyTorch's round-to-nearest-even float8_e4m3fn cast.  torch's cast
    does not saturate, so the range stops at 448."""
    lo = int(np.float32(2.0 ** -12).view(np.uint32))
    hi = int(np.float32(448.0).view(np.uint32))
    step = 1 << 24
    for start in range(lo, hi + 1, 3 * step):
        pats = np.arange(start, min(hi + 1, start + 3 * step), 3, dtype=np.uint32)
        for sign in (0, 0x80000000):
            vals = (pats | np.uint32(sign)).view(np.float32)
            ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            got = orc.e4m3_encode_array(vals)
            bad = np.nonzero(got != ref)[0]
            assert bad.size == 0, (hex(int(vals.view(np.uint32)[bad[0]])), got[bad[0]], ref[bad[0]])


@pytest.mark.slow
def test_encode_exhaustive_all_binary32(orc):
    """The bit-manipulation encoder equals the nearest-value-search encoder on
    all 2^32 binary32 patterns."""
    bad, first = orc.e4m3_exhaustive_check(0, 1 << 32, 1)
    assert bad == 0, "first mismatching pattern 0x%08x" % first


def test_encode_exhaustive_check_detects_mismatch(orc):
    """The search encoder is a real second opinion: it disagrees with a
    deliberately wrong rule (truncation) on ordinary values."""
    v = 1.0 + 2 ** -4 + 2 ** -6  # 1.078125 -> RNE 1.125 (0x39); truncation would give 1.0
    assert orc.e4m3_encode_by_search(v) == 0x39 == orc.e4m3_encode(v)
