"""The chained MoE decode on the GPU: masked GEMM1 -> SwiGLU fused with the
1x128 requantization -> masked GEMM2, against the oracle.

The SwiGLU kernel's output (codes and scales of h) is compared bit for bit
with the oracle's SwiGLU (double, rounded once to bf16) followed by its 1x128
quantization, on the same bf16 input.  The chain's GEMM2 output is compared
within the GEMM tolerance with the oracle run on the GPU's own GEMM1 output.
"""
import numpy as np
import pytest
import torch

import oracle
import fp8_fine_grained_quant_b200 as fq
import workloads as wl
from parity import assert_gemm_close, bf16_bits_of, bytes_of, to_torch_bf16

pytestmark = pytest.mark.gpu
TILE = 128


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _c1(rng, rows, inter):
    """GEMM1-like [gate | up] rows plus the edge values of the SwiGLU: zeros,
    gates far below the FP32 exp range, huge magnitudes, tiny products."""
    g = rng.standard_normal((rows, inter)) * np.exp(rng.uniform(-4, 3, (rows, inter)))
    u = rng.standard_normal((rows, inter)) * np.exp(rng.uniform(-4, 4, (rows, inter)))
    specials_g = [0.0, -0.0, -88.0, -89.0, -100.0, -1e30, 1e30, 100.0, 3e38, -3e38, 1e-30, -87.5]
    specials_u = [1.0, -2.0, 1.0, 3.0, -1.0, 2.0, 2.0, -5.0, 0.5, 0.5, 1e-30, 1e3]  # h stays finite
    for k, (a, b) in enumerate(zip(specials_g, specials_u)):
        g[k % rows, (7 * k) % inter] = a
        u[k % rows, (7 * k) % inter] = b
    return wl.bf16_bits(np.concatenate([g, u], axis=1).astype(np.float32))


@pytest.mark.parametrize("rows,inter", [(1, 128), (300, 256), (64, 2048), (1024, 512)])
def test_swiglu_quant_matches_oracle(dev, rows, inter):
    rng = np.random.default_rng(rows + inter)
    c1 = _c1(rng, rows, inter)
    qh, sh = fq.fp8_swiglu_quant_1x128(to_torch_bf16(c1, dev))
    torch.cuda.synchronize(dev)
    assert fq.get_device_error(device=dev) == fq.OK
    oq, os_ = oracle.quant_act_1x128(oracle.swiglu_bf16(c1))
    assert np.array_equal(sh.cpu().numpy().view(np.uint32), os_.view(np.uint32))
    assert np.array_equal(bytes_of(qh).reshape(rows, inter), oq)


def test_swiglu_quant_masked_rows_untouched(dev):
    E, cap, inter = 3, 256, 256
    rng = np.random.default_rng(3)
    c1 = _c1(rng, E * cap, inter).reshape(E, cap, 2 * inter)
    masked_m = np.array([0, 130, 256], dtype=np.int32)
    qh = torch.full((E, cap, inter), 0x5A, dtype=torch.uint8, device=dev)
    sh = torch.full((E, cap, inter // TILE), -3.0, dtype=torch.float32, device=dev)
    fq.fp8_swiglu_quant_1x128(to_torch_bf16(c1, dev), masked_m=torch.from_numpy(masked_m).to(dev), qh=qh, sh=sh)
    torch.cuda.synchronize(dev)
    assert fq.get_device_error(device=dev) == fq.OK
    q, s = qh.cpu().numpy(), sh.cpu().numpy()
    for e in range(E):
        m = int(masked_m[e])
        assert np.all(q[e, m:] == 0x5A) and np.all(s[e, m:] == -3.0)
        if m:
            oq, os_ = oracle.quant_act_1x128(oracle.swiglu_bf16(c1[e, :m]))
            assert np.array_equal(q[e, :m], oq)
            assert np.array_equal(s[e, :m].view(np.uint32), os_.view(np.uint32))


def test_masked_chain(dev):
    """GEMM1 -> SwiGLU + requantization -> GEMM2 for a small masked batch."""
    E, cap, K1, inter, N2 = 4, 256, 512, 256, 384
    rng = np.random.default_rng(11)
    a = wl.bf16_bits(rng.standard_normal((E, cap, K1)).astype(np.float32))
    b1 = wl.bf16_bits((0.05 * rng.standard_normal((E, 2 * inter, K1))).astype(np.float32))
    b2 = wl.bf16_bits((0.05 * rng.standard_normal((E, N2, inter))).astype(np.float32))
    masked_m = np.array([5, 0, 256, 129], dtype=np.int32)
    mm = torch.from_numpy(masked_m).to(dev)
    qa, sa = fq.fp8_quant_act_1x128(to_torch_bf16(a.reshape(E * cap, K1), dev))
    qb1, sb1 = fq.fp8_quant_w_128x128(to_torch_bf16(b1, dev))
    c1 = torch.zeros((E, cap, 2 * inter), dtype=torch.bfloat16, device=dev)
    fq.fp8_grouped_gemm_masked(qa.view(E, cap, K1), sa.view(E, cap, K1 // TILE), qb1, sb1, mm, out=c1)
    qh, sh = fq.fp8_swiglu_quant_1x128(c1, masked_m=mm)
    qb2, sb2 = fq.fp8_quant_w_128x128(to_torch_bf16(b2, dev))
    c2 = torch.zeros((E, cap, N2), dtype=torch.bfloat16, device=dev)
    fq.fp8_grouped_gemm_masked(qh, sh, qb2, sb2, mm, out=c2)
    torch.cuda.synchronize(dev)
    assert fq.get_device_error(device=dev) == fq.OK

    c1_bits = bf16_bits_of(c1)
    oqa, osa = oracle.quant_act_1x128(a.reshape(E * cap, K1))
    oqb1, osb1 = oracle.quant_w_128x128(b1)
    ref1 = oracle.grouped_masked(oqa.reshape(E, cap, K1), osa.reshape(E, cap, K1 // TILE), oqb1, osb1, masked_m)
    oqb2, osb2 = oracle.quant_w_128x128(b2)
    c2_bits = bf16_bits_of(c2)
    for e in range(E):
        m = int(masked_m[e])
        if not m:
            continue
        assert_gemm_close(c1_bits[e, :m], ref1[e, :m], "GEMM1 expert %d" % e)
        # the oracle's SwiGLU and requantization of the GPU's own GEMM1 output
        oqh, osh = oracle.quant_act_1x128(oracle.swiglu_bf16(c1_bits[e, :m]))
        ref2 = oracle.gemm_blockscaled(oqh, osh, oqb2[e], osb2[e])
        assert_gemm_close(c2_bits[e, :m], ref2, "GEMM2 expert %d" % e)
