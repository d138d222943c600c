"""Pins for the oracle's 1x128 activation and 128x128 weight quantizers (CPU).

What fixes the answer:
* hand-computed worked examples (tests/golden/quant_worked_examples.txt);
* the grouping geometry of Figure 7 (a) in "The Insider Secrets Of Deepseek
  Discovered" (one scale per token per 128 channels; one per 128x128 weight
  block): a single outlier changes exactly its own group;
* the scaling rule of the same passage (largest magnitude -> FP8 maximum):
  the amax element encodes to +-448, every code decodes to |v| <= 448, s > 0,
  an all-zero group gets s = 1, a group whose amax is already 448 gets s = 1
  and q equal to PyTorch's own E4M3 cast of x.
"""
import numpy as np
import pytest
import torch

from conftest import golden_lines, hexfloat
from workloads import bf16_bits, bf16_to_f32, tiny_dense

TILE = 128


def _bits(values):
    return bf16_bits(np.asarray(values, dtype=np.float32))


def _parse_worked():
    ex = {"act": {}, "act2": {}, "w": {}}
    for tok in golden_lines("quant_worked_examples.txt"):
        kind = tok[0]
        if kind in ("act", "act2") and tok[1] == "K":
            ex[kind]["K"] = int(tok[2])
            ex[kind]["scales"], ex[kind]["elems"] = {}, []
        elif kind in ("act_scale", "act2_scale"):
            ex[kind[:-6]]["scales"][int(tok[1])] = hexfloat(tok[2])
        elif kind in ("act", "act2"):
            ex[kind]["elems"].append((int(tok[1]), hexfloat(tok[2]), int(tok[3], 16)))
        elif kind == "w" and tok[1] == "N":
            ex["w"].update(N=int(tok[2]), K=int(tok[4]), scales={}, elems=[])
        elif kind == "w_scale":
            ex["w"]["scales"][(int(tok[1]), int(tok[2]))] = hexfloat(tok[3])
        elif kind == "w":
            ex["w"]["elems"].append((int(tok[1]), int(tok[2]), hexfloat(tok[3]), int(tok[4], 16)))
    return ex


@pytest.mark.parametrize("which", ["act", "act2"])
def test_worked_activation_examples(orc, which):
    ex = _parse_worked()[which]
    K = ex["K"]
    x = np.zeros((1, K), dtype=np.float32)
    for k, v, _ in ex["elems"]:
        x[0, k] = v
    xb = _bits(x)
    assert np.array_equal(bf16_to_f32(xb), x), "worked-example inputs must be bf16-exact"
    q, s = orc.quant_act_1x128(xb)
    assert s.shape == (1, K // TILE)
    for kb, sv in ex["scales"].items():
        assert s[0, kb] == np.float32(sv), (kb, float(s[0, kb]).hex(), sv)
    expect = np.zeros(K, dtype=np.uint8)
    for k, _, code in ex["elems"]:
        expect[k] = code
    assert np.array_equal(q[0], expect), np.nonzero(q[0] != expect)


def test_worked_weight_example(orc):
    ex = _parse_worked()["w"]
    N, K = ex["N"], ex["K"]
    w = np.zeros((N, K), dtype=np.float32)
    for r, c, v, _ in ex["elems"]:
        w[r, c] = v
    q, s = orc.quant_w_128x128(_bits(w))
    assert s.shape == (N // TILE, K // TILE)
    for (nb, kb), sv in ex["scales"].items():
        assert s[nb, kb] == np.float32(sv)
    expect = np.zeros((N, K), dtype=np.uint8)
    for r, c, _, code in ex["elems"]:
        expect[r, c] = code
    assert np.array_equal(q, expect)


def test_zero_groups_get_unit_scale(orc):
    q, s = orc.quant_act_1x128(np.zeros((3, 256), dtype=np.uint16))
    assert np.all(s == 1.0) and np.all(q == 0)
    q, s = orc.quant_w_128x128(np.zeros((2, 128, 256), dtype=np.uint16))
    assert np.all(s == 1.0) and np.all(q == 0)
    # -0.0 inputs keep their sign through the unit scale
    q, s = orc.quant_act_1x128(np.full((1, 128), 0x8000, dtype=np.uint16))
    assert np.all(s == 1.0) and np.all(q == 0x80)


def test_amax_448_groups_reduce_to_plain_cast(orc):
    """amax == 448 gives s == 1, so q must equal PyTorch's RNE E4M3 cast of x."""
    rng = np.random.default_rng(11)
    x = rng.uniform(-447.0, 447.0, size=(4, 512)).astype(np.float32)
    x[:, ::TILE] = 448.0
    xb = _bits(x)
    q, s = orc.quant_act_1x128(xb)
    assert np.all(s == 1.0)
    ref = torch.from_numpy(bf16_to_f32(xb)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)
    w = rng.uniform(-447.0, 447.0, size=(256, 256)).astype(np.float32)
    w[::TILE, ::TILE] = -448.0
    wb = _bits(w)
    q, s = orc.quant_w_128x128(wb)
    assert np.all(s == 1.0)
    ref = torch.from_numpy(bf16_to_f32(wb)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)


def test_invariants_on_outlier_workload(orc):
    d = tiny_dense()
    table = orc.e4m3_decode_table()
    for q, s, x, groups in (
        (*orc.quant_act_1x128(d.a), d.a, "act"),
        (*orc.quant_w_128x128(d.b), d.b, "w"),
    ):
        xf = bf16_to_f32(x)
        v = table[q]
        assert np.all(np.isfinite(v)) and np.all(np.abs(v) <= 448.0)
        assert np.all(s > 0)
        if groups == "act":
            g = np.abs(xf).reshape(xf.shape[0], -1, TILE)
            amax = g.max(axis=2)
            qa = q.reshape(g.shape)
            hit = g == amax[..., None]
            assert np.all((qa[hit] & 0x7F) == 0x7E), "amax element must encode to +-448"
            assert np.array_equal(s, (amax / np.float32(448.0)).astype(np.float32))
            # sign preserved
            xs = xf.reshape(g.shape)
            nz = xs != 0
            assert np.all((qa[nz & (xs < 0)] & 0x80) == 0x80)
        else:
            N, K = xf.shape
            g = np.abs(xf).reshape(N // TILE, TILE, K // TILE, TILE)
            amax = g.max(axis=(1, 3))
            assert np.array_equal(s, (amax / np.float32(448.0)).astype(np.float32))
            qb = q.reshape(g.shape)
            hit = g == amax[:, None, :, None]
            assert np.all((qb[hit] & 0x7F) == 0x7E)


def test_dequantized_error_bound(orc):
    """|decode(q)*s - x| is at most half an E4M3 step of x/s (plus the f32
    rounding of the quotient): relative 2^-4 for normals, 2^-10*s absolute
    in the subnormal range."""
    d = tiny_dense(seed=5)
    q, s = orc.quant_act_1x128(d.a)
    table = orc.e4m3_decode_table()
    x = bf16_to_f32(d.a).astype(np.float64)
    sv = np.repeat(s.astype(np.float64), TILE, axis=1)
    y = x / sv
    deq = table[q]
    err = np.abs(deq - y)
    bound = np.maximum(np.abs(y) * 2.0 ** -4, 2.0 ** -10) * (1 + 1e-6)
    assert np.all(err <= bound)


def test_single_outlier_changes_only_its_group_act(orc):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 640)).astype(np.float32)
    base_q, base_s = orc.quant_act_1x128(_bits(x))
    m, k = 2, 300
    x2 = x.copy()
    x2[m, k] = 1000.0
    q, s = orc.quant_act_1x128(_bits(x2))
    ds = np.argwhere(s != base_s)
    assert ds.tolist() == [[m, k // TILE]]
    dq = np.argwhere(q != base_q)
    assert np.all(dq[:, 0] == m) and np.all(dq[:, 1] // TILE == k // TILE)
    assert len(dq) > 64  # the whole tile is rescaled, not just the outlier


def test_single_outlier_changes_only_its_group_w(orc):
    rng = np.random.default_rng(4)
    w = (0.02 * rng.standard_normal((384, 512))).astype(np.float32)
    base_q, base_s = orc.quant_w_128x128(_bits(w))
    r, c = 200, 77
    w2 = w.copy()
    w2[r, c] = 5.0
    q, s = orc.quant_w_128x128(_bits(w2))
    assert np.argwhere(s != base_s).tolist() == [[r // TILE, c // TILE]]
    dq = np.argwhere(q != base_q)
    assert np.all(dq[:, 0] // TILE == r // TILE) and np.all(dq[:, 1] // TILE == c // TILE)
    assert len(dq) > 8000


def test_weight_batch_matches_per_matrix(orc):
    rng = np.random.default_rng(8)
    w = _bits(rng.standard_normal((3, 256, 384)).astype(np.float32))
    q, s = orc.quant_w_128x128(w)
    for g in range(3):
        qg, sg = orc.quant_w_128x128(np.ascontiguousarray(w[g]))
        assert np.array_equal(q[g], qg) and np.array_equal(s[g], sg)


def test_bf16_generator_rounding_matches_torch():
    """The input generator's float32 -> bf16 conversion is torch's RNE cast."""
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(1 << 16) * np.exp(rng.uniform(-20, 20, 1 << 16))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bf16_bits(x), ref)


def test_rejects_bad_shapes(orc):
    with pytest.raises(ValueError):
        orc.quant_w_128x128(np.zeros((100, 128), dtype=np.uint16))


# --------------------------------------------------------------------------- delayed scaling (given scale)
def _golden_bf16_encodings():
    out = []
    for tok in golden_lines("e4m3_encodings.txt"):
        if tok[0] == "decode" or tok[0].lower() == "nan":
            continue
        v = np.float32(hexfloat(tok[0]))
        b = bf16_bits(np.array([v], dtype=np.float32))
        if bf16_to_f32(b)[0] == v:  # exactly a bf16 value
            out.append((b[0], int(tok[1], 16)))
    return out


def test_quant_with_scale_golden_encodings(orc):
    """With s = 1 the codes are the hand-computed encodings; with s = 2^-3 and
    inputs scaled by 2^-3 (exact in bf16) they are the same codes."""
    cases = _golden_bf16_encodings()
    assert len(cases) >= 15
    bits = np.array([b for b, _ in cases], dtype=np.uint16)
    codes = np.array([c for _, c in cases], dtype=np.uint8)
    assert np.array_equal(orc.quant_with_scale(bits, 1.0), codes)
    scaled = bf16_bits(bf16_to_f32(bits) * np.float32(0.125))
    assert np.array_equal(bf16_to_f32(scaled), bf16_to_f32(bits) * np.float32(0.125))
    assert np.array_equal(orc.quant_with_scale(scaled, 0.125), codes)


def test_quant_with_scale_saturates_beyond_448s(orc):
    x = bf16_bits(np.array([[1e-3, -1e-3, 5.0, -7.0, 0.0]], dtype=np.float32))
    q = orc.quant_with_scale(x, 1e-6)  # every nonzero |x| / s is at least 1000 > 448
    assert list(q[0]) == [0x7E, 0xFE, 0x7E, 0xFE, 0x00]


def test_quant_with_scale_at_current_amax_is_per_tensor(orc):
    d = tiny_dense()
    q_t, s_t = orc.quant_tensor(d.a)
    assert np.array_equal(orc.quant_with_scale(d.a, s_t), q_t)


def test_scaling_study_orders_the_schemes(orc):
    """On the outlier workload: fine-grained groups beat one scale per tensor,
    and a delayed scale that has not seen a new outlier clips it (large
    error) while the fine-grained scheme is unaffected."""
    from oracle.scaling_accuracy import study
    d = tiny_dense()
    rows = np.arange(d.a.shape[0], dtype=np.int64)
    r = {x["name"]: x for x in study(d.a, d.b, rows)}
    fine = r["fine-grained 1x128 / 128x128, online"]
    tensor = r["per-tensor, online"]
    spike_delayed = r["per-tensor, delayed (new outlier at 4x the history max)"]
    spike_fine = r["fine-grained, online, same new outlier"]
    assert fine["act_err"] < tensor["act_err"] and fine["fro_rel"] < tensor["fro_rel"]
    assert spike_delayed["fro_rel"] > 3 * spike_fine["fro_rel"]
    assert spike_fine["fro_rel"] < 1.1 * fine["fro_rel"]


# --------------------------------------------------------------------------- power-of-two (UE8M0) scales
@pytest.mark.parametrize("amax,expect", [
    (448.0, 1.0),                 # 448 * 2^0 >= 448, and 448 * 2^-1 < 448
    (450.0, 2.0),                 # the next bf16 above 448
    (1.0, 2.0 ** -8),             # 448 / 256 = 1.75 >= 1 > 0.875 = 448 / 512
    (224.0, 0.5),                 # exactly 448 * 2^-1
    (0.0, 1.0),
    (float(np.float32(3.3895313892515355e38)), 2.0 ** 120),   # largest bf16
    (2.0 ** -133, 2.0 ** -127),   # smallest bf16 subnormal: exponent clamped to the E8M0 range
])
def test_ue8m0_scale_hand_cases(orc, amax, expect):
    x = np.zeros((1, 128), dtype=np.float32)
    x[0, 17] = amax
    x[0, 40] = -amax / 3
    q, s = orc.quant_act_1x128_ue8m0(bf16_bits(x))
    assert s[0, 0] == np.float32(expect)
    if amax > 0:
        assert orc.e4m3_decode(q[0, 17]) * float(s[0, 0]) <= amax * 1.0625  # within an E4M3 step, never clipped


def test_ue8m0_scales_are_the_least_power_of_two_cover(orc):
    d = tiny_dense()
    for quant, per_group in ((orc.quant_act_1x128_ue8m0, "act"), (orc.quant_w_128x128_ue8m0, "w")):
        src = d.a if per_group == "act" else d.b
        q, s = quant(src)
        f = bf16_to_f32(src).astype(np.float64)
        if per_group == "act":
            amax = np.abs(f).reshape(f.shape[0], -1, 128).max(axis=2)
        else:
            n, k = f.shape
            amax = np.abs(f).reshape(n // 128, 128, k // 128, 128).max(axis=(1, 3))
        s64 = s.astype(np.float64)
        mant, _ = np.frexp(s64)
        assert np.all(mant == 0.5), "every scale is a power of two"
        assert np.all(448.0 * s64 >= amax)
        assert np.all((224.0 * s64 < amax) | (amax == 0))
        # no saturation: every code is exactly the RNE code of x / s (an exact quotient)
        reps = np.repeat(s64, 128, axis=1) if per_group == "act" else np.repeat(np.repeat(s64, 128, 0), 128, 1)
        expect = orc.e4m3_encode_array((f / reps).astype(np.float32))
        assert np.array_equal(q, expect.reshape(q.shape))


def test_ue8m0_vs_fp32_scales(orc):
    """The power-of-two scale is the fp32 scale rounded up to a power of two."""
    d = tiny_dense()
    _, s2 = orc.quant_act_1x128_ue8m0(d.a)
    _, s32 = orc.quant_act_1x128(d.a)
    assert np.all(s2 >= s32) and np.all(s2 < 2 * s32)


def test_ue8m0_all_ones_gemm_is_exact(orc):
    """All-ones operands: every scale is 2^-8, every code is 256 (0x78), and the
    block-scaled product is exactly K (no rounding anywhere)."""
    M, N, K = 4, 256, 640
    a = np.full((M, K), 0x3F80, dtype=np.uint16)
    b = np.full((N, K), 0x3F80, dtype=np.uint16)
    qa, sa = orc.quant_act_1x128_ue8m0(a)
    qb, sb = orc.quant_w_128x128_ue8m0(b)
    assert np.all(qa == 0x78) and np.all(sa == 2.0 ** -8) and np.all(sb == 2.0 ** -8)
    assert np.all(orc.gemm_blockscaled(qa, sa, qb, sb) == float(K))
