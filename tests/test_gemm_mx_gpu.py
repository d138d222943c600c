"""Block-scaled GEMM with power-of-two scales applied by the tensor cores,
against the oracle's float64 product on the same power-of-two quantization.
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


def _mx_case(dev, a, b, rows=None):
    qa, sa = fq.fp8_quant_act_1x128_ue8m0(to_torch_bf16(a, dev))
    qb, sb = fq.fp8_quant_w_128x128_ue8m0(to_torch_bf16(b, dev))
    sfa, sfb = fq.fp8_mx_scales_act(sa), fq.fp8_mx_scales_w(sb)
    c = fq.fp8_gemm_mx(qa, sfa, qb, sfb)
    torch.cuda.synchronize(dev)
    assert fq.get_device_error(device=dev) == fq.OK
    oqa, osa = oracle.quant_act_1x128_ue8m0(a)
    oqb, osb = oracle.quant_w_128x128_ue8m0(b)
    ref = oracle.gemm_blockscaled(oqa, osa, oqb, osb, rows=rows)
    got = bf16_bits_of(c)
    return (got if rows is None else got[rows]), ref, sfa


def test_scale_atoms(dev):
    """The converters' atoms hold each row's E8M0 code at 16*m0 + 4*m1 + j."""
    M, K = 300, 384
    rng = np.random.default_rng(1)
    a = wl.bf16_bits((rng.standard_normal((M, K)) * np.exp(rng.uniform(-20, 20, (M, 1)))).astype(np.float32))
    _, sa = fq.fp8_quant_act_1x128_ue8m0(to_torch_bf16(a, dev))
    atoms = fq.fp8_mx_scales_act(sa).cpu().numpy()
    codes = (sa.cpu().numpy().view(np.uint32) >> 23) & 0xFF
    for mt in range(atoms.shape[0]):
        for m in range(128):
            row = mt * 128 + m
            want = codes[row] if row < M else np.full(K // TILE, 127)
            got = atoms[mt, :, 16 * (m % 32) + 4 * (m // 32):16 * (m % 32) + 4 * (m // 32) + 4]
            assert np.all(got == np.asarray(want)[:, None])


@pytest.mark.parametrize("M,N,K", [(128, 128, 128), (300, 256, 512), (256, 384, 1024), (1, 128, 256)])
def test_gemm_mx_matches_oracle(dev, M, N, K):
    rng = np.random.default_rng(M + N + K)
    a = wl.bf16_bits((rng.standard_normal((M, K)) * np.exp(rng.standard_normal(K))).astype(np.float32))
    b = wl.bf16_bits((0.02 * rng.standard_normal((N, K))).astype(np.float32))
    got, ref, _ = _mx_case(dev, a, b)
    assert_gemm_close(got, ref, "gemm_mx %dx%dx%d" % (M, N, K))


def test_gemm_mx_full_size_sampled_rows(dev):
    d = wl.dense_fprop()
    rows = wl.quad_rows(np.random.default_rng(12), d.M).tolist()
    got, ref, _ = _mx_case(dev, d.a, d.b, rows=rows)
    assert_gemm_close(got, ref, "gemm_mx dense_fprop, %d rows" % len(rows))


def _mx_grouped_operands(dev, a, b):
    qa, sa = fq.fp8_quant_act_1x128_ue8m0(to_torch_bf16(a.reshape(-1, a.shape[-1]), dev))
    qb, sb = fq.fp8_quant_w_128x128_ue8m0(to_torch_bf16(b, dev))
    return qa, fq.fp8_mx_scales_act(sa), qb, fq.fp8_mx_scales_w(sb)


def test_grouped_mx_contiguous_matches_oracle(dev):
    d = wl.moe_contiguous(tokens=96, topk=4, E=6, N=384, K=512, seed=21)
    qa, sfa, qb, sfb = _mx_grouped_operands(dev, d.a, d.b)
    mi = torch.from_numpy(d.m_indices).to(dev)
    c = fq.fp8_grouped_gemm_mx_contiguous(qa, sfa, qb, sfb, mi)
    torch.cuda.synchronize(dev)
    assert fq.get_device_error(device=dev) == fq.OK
    oqa, osa = oracle.quant_act_1x128_ue8m0(d.a)
    oqb, osb = oracle.quant_w_128x128_ue8m0(d.b)
    ref = oracle.grouped_contiguous(oqa, osa, oqb, osb, d.m_indices)
    assert_gemm_close(bf16_bits_of(c), ref, "grouped mx contiguous")


def test_grouped_mx_masked_matches_oracle(dev):
    E, cap, N, K = 4, 256, 384, 512
    rng = np.random.default_rng(33)
    a = wl.bf16_bits(rng.standard_normal((E, cap, K)).astype(np.float32))
    b = wl.bf16_bits((0.02 * rng.standard_normal((E, N, K))).astype(np.float32))
    masked_m = np.array([5, 0, 256, 129], dtype=np.int32)
    qa, sfa, qb, sfb = _mx_grouped_operands(dev, a, b)
    out = torch.full((E, cap, N), -5.0, dtype=torch.bfloat16, device=dev)
    fq.fp8_grouped_gemm_mx_masked(qa.view(E, cap, K), sfa, qb, sfb, torch.from_numpy(masked_m).to(dev), out=out)
    torch.cuda.synchronize(dev)
    assert fq.get_device_error(device=dev) == fq.OK
    oqa, osa = oracle.quant_act_1x128_ue8m0(a.reshape(E * cap, K))
    oqb, osb = oracle.quant_w_128x128_ue8m0(b)
    ref = oracle.grouped_masked(oqa.reshape(E, cap, K), osa.reshape(E, cap, K // TILE), oqb, osb, masked_m)
    got = bf16_bits_of(out)
    for e in range(E):
        m = int(masked_m[e])
        assert np.all(got[e, m:] == 0xC0A0)             # bf16 -5.0 untouched
        if m:
            assert_gemm_close(got[e, :m], ref[e, :m], "grouped mx masked expert %d" % e)
