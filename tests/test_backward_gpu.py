"""GPU kernels of the backward GEMMs' operands vs the oracle (bit for bit).

Dgrad (dX = dY W) is the forward GEMM on W's block-quantized codes and scales
transposed; Wgrad (dW = dY^T X) needs both operands grouped along tokens
(128x1 tiles).  "The Insider Secrets Of Deepseek Discovered", Figure 6: all
three GEMMs of a linear layer run in FP8.
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


def _bits(rng, shape, scale=1.0, outliers=0, chan=False):
    x = (scale * rng.standard_normal(shape)).astype(np.float32)
    if chan:
        x *= np.exp(rng.standard_normal(shape[-1])).astype(np.float32)
    if outliers:
        idx = rng.choice(x.size, size=outliers, replace=False)
        x.reshape(-1)[idx] = np.where(rng.random(outliers) < 0.5, -200.0, 200.0)
    return wl.bf16_bits(x)


# (3000, 7168): 24 x 56 = 1344 blocks, about 4.5 per CTA of the persistent
# grid (2 per SM), so every CTA cycles through all three shared stages
@pytest.mark.parametrize("M,K", [(128, 128), (256, 384), (200, 256), (1, 128), (1000, 640), (3000, 7168)])
def test_token_axis_quant_matches_oracle(dev, M, K):
    rng = np.random.default_rng(M * 7 + K)
    x = _bits(rng, (M, K), outliers=max(1, M * K // 5000), chan=True)
    if M > 10:
        x[3, :] = 0      # a zero token
        x[:, 5] = 0      # a zero channel: scale 1
    q, s = fq.fp8_quant_act_128x1(to_torch_bf16(x, dev))
    torch.cuda.synchronize(dev)
    oq, os_ = oracle.quant_act_128x1(x)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), os_.view(np.uint32))
    assert np.array_equal(bytes_of(q).reshape(M, K), oq)


@pytest.mark.parametrize("token_contiguous", [False, True])
def test_token_axis_quant_every_bf16_amax(dev, token_contiguous):
    """Every 16th finite non-negative bf16 value as the amax of one group."""
    amax_bits = np.arange(0, 0x7F80, 16, dtype=np.uint32)
    a = (amax_bits << 16).view(np.float32)
    rng = np.random.default_rng(5)
    g = a.size                                    # 2040 groups = channels
    x = (a[None, :] * rng.random((TILE, g), dtype=np.float32)
         * np.where(rng.random((TILE, g)) < 0.5, -1.0, 1.0).astype(np.float32))
    xb = wl.bf16_bits(x)
    xb[7, :] = amax_bits.astype(np.uint16)        # the amax of each channel's group
    K = (g + TILE - 1) // TILE * TILE
    xb = np.pad(xb, ((0, 0), (0, K - g)))
    oq, os_ = oracle.quant_act_128x1(xb)
    if token_contiguous:
        qt, s = fq.fp8_quant_act_128x1_t(to_torch_bf16(xb, dev), Mp=TILE)
        torch.cuda.synchronize(dev)
        assert np.array_equal(bytes_of(qt).reshape(K, TILE), np.ascontiguousarray(oq.T))
    else:
        q, s = fq.fp8_quant_act_128x1(to_torch_bf16(xb, dev))
        torch.cuda.synchronize(dev)
        assert np.array_equal(bytes_of(q).reshape(xb.shape), oq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), os_.view(np.uint32))


@pytest.mark.parametrize("shape", [(128, 128), (256, 384), (3, 128, 256)])
def test_weight_transpose(dev, shape):
    rng = np.random.default_rng(sum(shape))
    w = _bits(rng, shape, scale=0.02)
    q, s = fq.fp8_quant_w_128x128(to_torch_bf16(w, dev))
    qt, st = fq.fp8_transpose_w_128x128(q, s)
    torch.cuda.synchronize(dev)
    qn, sn = bytes_of(q).reshape(shape), s.cpu().numpy()
    assert np.array_equal(bytes_of(qt).reshape(shape[:-2] + (shape[-1], shape[-2])), np.swapaxes(qn, -1, -2))
    assert np.array_equal(st.cpu().numpy(), np.swapaxes(sn, -1, -2))


@pytest.mark.parametrize("M,N,K", [(256, 256, 384), (200, 512, 256)])
def test_dgrad_through_the_forward_gemm(dev, M, N, K):
    """dX = dY W: 1x128 tiles of dY, W's blocks transposed, the forward GEMM."""
    rng = np.random.default_rng(M + N + K)
    dy = _bits(rng, (M, N), outliers=4, chan=True)
    w = _bits(rng, (N, K), scale=0.02)
    q_dy, s_dy = fq.fp8_quant_act_1x128(to_torch_bf16(dy, dev))
    q_w, s_w = fq.fp8_quant_w_128x128(to_torch_bf16(w, dev))
    qt, st = fq.fp8_transpose_w_128x128(q_w, s_w)
    dx = fq.fp8_gemm_blockscaled(q_dy, s_dy, qt, st)
    torch.cuda.synchronize(dev)
    assert fq.get_device_error(device=dev) == fq.OK
    oq_dy, os_dy = oracle.quant_act_1x128(dy)
    oq_w, os_w = oracle.quant_w_128x128(w)
    ref = oracle.dgrad(oq_dy, os_dy, oq_w, os_w)
    assert_gemm_close(bf16_bits_of(dx), ref, "dgrad %dx%dx%d" % (M, N, K))


def _pad_tokens(x, Mp):
    return np.pad(x, ((0, Mp - x.shape[0]), (0, 0)))


@pytest.mark.parametrize("M,K,pad", [(128, 128, 128), (256, 384, 512), (200, 256, 128), (1, 128, 512),
                                     (1000, 640, 128), (1000, 640, 512), (3000, 7168, 512)])
def test_token_contiguous_quant_matches_oracle(dev, M, K, pad):
    """Token-axis groups with the codes written token-contiguous: qt[k, m] is
    the code of x[m, k]; padding tokens (m >= M) get code 0 and groups made
    only of padding scale 1."""
    rng = np.random.default_rng(M * 11 + K)
    x = _bits(rng, (M, K), outliers=max(1, M * K // 5000), chan=True)
    if M > 10:
        x[3, :] = 0
        x[:, 5] = 0
    Mp = -(-M // pad) * pad
    qt, s = fq.fp8_quant_act_128x1_t(to_torch_bf16(x, dev), Mp=Mp)
    torch.cuda.synchronize(dev)
    assert fq.get_device_error(device=dev) == fq.OK
    oq, os_ = oracle.quant_act_128x1(_pad_tokens(x, Mp))
    assert np.array_equal(oq[M:], np.zeros_like(oq[M:]))
    assert np.all(os_[-(-M // TILE):] == 1.0)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), os_.view(np.uint32))
    assert np.array_equal(bytes_of(qt).reshape(K, Mp), np.ascontiguousarray(oq.T))


@pytest.mark.parametrize("M,N,K", [(256, 256, 384), (300, 128, 256), (1024, 512, 640), (128, 128, 128)])
def test_wgrad_matches_oracle(dev, M, N, K):
    """dW = dY^T X over tokens, both operands in token-axis groups."""
    rng = np.random.default_rng(M + 3 * N + 7 * K)
    dy = _bits(rng, (M, N), outliers=4, chan=True)
    x = _bits(rng, (M, K), outliers=4, chan=True)
    q_dy_t, s_dy = fq.fp8_quant_act_128x1_t(to_torch_bf16(dy, dev))
    q_x_t, s_x = fq.fp8_quant_act_128x1_t(to_torch_bf16(x, dev))
    dw = fq.fp8_gemm_wgrad(q_dy_t, s_dy, q_x_t, s_x)
    torch.cuda.synchronize(dev)
    assert fq.get_device_error(device=dev) == fq.OK
    # zero tokens up to the padded count change neither a group's amax nor the sums
    Mp = -(-M // 512) * 512
    oq_dy, os_dy = oracle.quant_act_128x1(_pad_tokens(dy, Mp))
    oq_x, os_x = oracle.quant_act_128x1(_pad_tokens(x, Mp))
    ref = oracle.wgrad(oq_dy, os_dy, oq_x, os_x)
    assert_gemm_close(bf16_bits_of(dw), ref, "wgrad %dx%dx%d" % (M, N, K))


def test_wgrad_full_size_sampled_rows(dev):
    """The dense_fprop layer's weight gradient: dY and X [4096, 7168], dW
    [7168, 7168] over 4096 tokens; from every 128-row tile of dW a row in
    each 32-row quad (every epilogue warp's rows), against the oracle."""
    d = wl.dense_fprop()
    rng = np.random.default_rng(9)
    dy = _bits(rng, d.a.shape, chan=True)
    x = d.a
    q_dy_t, s_dy = fq.fp8_quant_act_128x1_t(to_torch_bf16(dy, dev))
    q_x_t, s_x = fq.fp8_quant_act_128x1_t(to_torch_bf16(x, dev))
    dw = fq.fp8_gemm_wgrad(q_dy_t, s_dy, q_x_t, s_x)
    torch.cuda.synchronize(dev)
    assert fq.get_device_error(device=dev) == fq.OK
    N = dy.shape[1]
    rows = wl.quad_rows(np.random.default_rng(10), N).tolist()
    oq_dy, os_dy = oracle.quant_act_128x1(dy)
    oq_x, os_x = oracle.quant_act_128x1(x)
    # the operands themselves are bit-exact (checked on the small shapes above); spot-check them here too
    assert np.array_equal(s_dy.cpu().numpy().view(np.uint32), os_dy.view(np.uint32))
    ref = oracle.wgrad(oq_dy, os_dy, oq_x, os_x, rows=rows)
    got = bf16_bits_of(dw)[rows]
    assert_gemm_close(got, ref, "wgrad full size, %d sampled rows" % len(rows))
