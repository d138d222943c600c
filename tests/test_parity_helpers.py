"""The GEMM tolerance check itself (CPU): correctly rounded results pass,
results off by more than the allowed pre-rounding error fail."""
import numpy as np
import torch

from parity import bf16_rne_f64, bf16_to_f64, gemm_errors, gemm_ok


def _bits(vals):
    return torch.from_numpy(np.asarray(vals, dtype=np.float64)).to(torch.float32).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def _bits_exact(vals64):
    """bf16 patterns of values that are already bf16-representable."""
    return _bits(vals64)


def test_bf16_rne_matches_torch_for_float32_inputs():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-30, 30, 100000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(bf16_rne_f64(x.astype(np.float64)), ref)


def test_bf16_rne_single_rounding():
    # 1 + 2^-8 + 2^-30: just above the midpoint of 1 and 1 + 2^-7 -> rounds up;
    # a float32 detour would first drop the 2^-30 and tie to even (1.0).
    x = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert bf16_rne_f64(np.array([x]))[0] == 1.0 + 2.0 ** -7


def _case(rel_shift, seed=1):
    rng = np.random.default_rng(seed)
    ref = rng.standard_normal(20000) * 3.0
    c = _bits_exact(bf16_rne_f64(ref * (1.0 + rel_shift)))
    return c, ref


def test_correct_rounding_passes_even_at_max_rounding_error():
    c, ref = _case(0.0)
    st = gemm_errors(c, ref)
    assert gemm_ok(st) and st["tol_used"] == 0.0 and st["not_correctly_rounded"] == 0
    assert st["out_max_rel"] > 3.5e-3  # raw bf16 rounding exceeds 2e-3


def test_small_pre_rounding_error_passes():
    st = gemm_errors(*_case(1.5e-3))
    assert gemm_ok(st), st


def test_pre_rounding_error_above_bound_fails():
    st = gemm_errors(*_case(2.6e-3))
    assert not gemm_ok(st), st


def test_absolute_bound_on_near_zero_elements():
    ref = np.array([100.0, -100.0, 1e-3, 0.0])
    rms = np.sqrt(np.mean(ref ** 2))
    ok = _bits_exact(bf16_rne_f64(np.array([100.0, -100.0, 1e-3 + 0.009 * rms, 0.0])))
    assert gemm_ok(gemm_errors(ok, ref))
    bad = _bits_exact(bf16_rne_f64(np.array([100.0, -100.0, 1e-3 + 0.02 * rms, 0.0])))
    assert not gemm_ok(gemm_errors(bad, ref))


def test_wrong_sign_and_nan_fail():
    c, ref = _case(0.0)
    c2 = c.copy()
    c2[7] ^= 0x8000
    assert not gemm_ok(gemm_errors(c2, ref))
    c3 = c.copy()
    c3[3] = 0x7FC0
    assert not gemm_ok(gemm_errors(c3, ref))
