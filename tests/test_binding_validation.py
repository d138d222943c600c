"""The Python binding checks every buffer size before any call (CPU only).

The C library is given pointers and sizes and trusts them, so a buffer that
is too small would be overrun on the device.  The binding therefore checks
dtypes, ranks, contiguity, the agreement of the operands' shapes and the
element count of every caller-supplied output first, then that every tensor
is a CUDA tensor on one device, and only then allocates and calls.  These
tests use host tensors: each bad size must be refused with its own message
before the device check, and well-formed host arguments must reach the device
check and be refused there.
"""
from types import SimpleNamespace

import pytest
import torch

import fp8_fine_grained_quant_b200 as fq

u8, f32, bf16, i32 = torch.uint8, torch.float32, torch.bfloat16, torch.int32


def z(*shape, dtype=u8):
    return torch.zeros(shape, dtype=dtype)


def dense(M=4, N=256, K=256):
    return [z(M, K), z(M, K // 128, dtype=f32), z(N, K), z(N // 128, K // 128, dtype=f32)]


@pytest.mark.parametrize("fn", [fq.fp8_gemm_blockscaled, fq.fp8_gemm_unpromoted_diag])
@pytest.mark.parametrize("mutate,match", [
    (lambda a: a.__setitem__(2, z(256, 384)), "differ in K"),
    (lambda a: a.__setitem__(2, z(200, 256)), "N = 200"),
    (lambda a: (a.__setitem__(0, z(4, 200)), a.__setitem__(2, z(256, 200))), "K = 200"),
    (lambda a: a.__setitem__(1, z(4, 3, dtype=f32)), "sa holds 12"),
    (lambda a: a.__setitem__(3, z(2, 1, dtype=f32)), "sb holds 2"),
    (lambda a: a.__setitem__(0, z(1, 4, 256)), "qa: expected"),
])
def test_dense_shapes(fn, mutate, match):
    args = dense()
    mutate(args)
    with pytest.raises(ValueError, match=match):
        fn(*args)


@pytest.mark.parametrize("fn", [fq.fp8_gemm_blockscaled, fq.fp8_gemm_unpromoted_diag])
def test_dense_out_size_and_dtype(fn):
    with pytest.raises(ValueError, match="out holds 1023"):
        fn(*dense(), out=z(1023, dtype=bf16))
    with pytest.raises(TypeError, match="out: dtype"):
        fn(*dense(), out=z(4, 256, dtype=f32))
    with pytest.raises(TypeError, match="sa: dtype"):
        a = dense()
        a[1] = a[1].double()
        fn(*a)
    with pytest.raises(ValueError, match="out must be contiguous"):
        fn(*dense(), out=z(256, 4, dtype=bf16).t())
    with pytest.raises(ValueError, match="CUDA tensor"):  # well formed: refused only for being on the host
        fn(*dense(), out=z(4, 256, dtype=bf16))


def contiguous(E=3, M_tot=384, N=256, K=256):
    return [z(M_tot, K), z(M_tot, K // 128, dtype=f32), z(E, N, K), z(E, N // 128, K // 128, dtype=f32),
            z(M_tot // 128, dtype=i32)]


@pytest.mark.parametrize("idx,bad,match", [
    (3, z(1, 2, 2, dtype=f32), "sb holds 4"),            # one expert's scales for three experts
    (4, z(4, dtype=i32), "m_indices holds 4"),
    (1, z(384, 1, dtype=f32), "sa holds 384"),
    (2, z(3, 256, 128), "differ in K"),
    (2, z(256, 256), "qb: expected"),
    (4, z(3, dtype=torch.int64), "m_indices: dtype"),
])
def test_contiguous_shapes(idx, bad, match):
    args = contiguous()
    args[idx] = bad
    with pytest.raises((ValueError, TypeError), match=match):
        fq.fp8_grouped_gemm_contiguous(*args)


def test_contiguous_rows_and_out():
    a = contiguous()
    a[0], a[1], a[4] = z(200, 256), z(200, 2, dtype=f32), z(1, dtype=i32)
    with pytest.raises(ValueError, match="M_tot = 200"):
        fq.fp8_grouped_gemm_contiguous(*a)
    with pytest.raises(ValueError, match="out holds 100"):
        fq.fp8_grouped_gemm_contiguous(*contiguous(), out=z(100, dtype=bf16))
    with pytest.raises(ValueError, match="CUDA tensor"):
        fq.fp8_grouped_gemm_contiguous(*contiguous(), out=z(384, 256, dtype=bf16))


def masked(E=2, cap=128, N=256, K=256):
    return [z(E, cap, K), z(E, cap, K // 128, dtype=f32), z(E, N, K), z(E, N // 128, K // 128, dtype=f32),
            z(E, dtype=i32)]


@pytest.mark.parametrize("idx,bad,match", [
    (2, z(3, 256, 256), "do not agree"),
    (1, z(2, 128, 1, dtype=f32), "sa holds 256"),
    (3, z(2, 1, 2, dtype=f32), "sb holds 4"),
    (4, z(3, dtype=i32), "masked_m holds 3"),
    (0, z(256, 256), "qa: expected"),
])
def test_masked_shapes(idx, bad, match):
    args = masked()
    args[idx] = bad
    with pytest.raises(ValueError, match=match):
        fq.fp8_grouped_gemm_masked(*args)


def test_masked_capacity_and_out():
    a = masked()
    a[0], a[1] = z(2, 100, 256), z(2, 100, 2, dtype=f32)
    with pytest.raises(ValueError, match="cap = 100"):
        fq.fp8_grouped_gemm_masked(*a)
    with pytest.raises(ValueError, match="out holds 65535"):
        fq.fp8_grouped_gemm_masked(*masked(), out=z(65535, dtype=bf16))
    with pytest.raises(ValueError, match="CUDA tensor"):
        fq.fp8_grouped_gemm_masked(*masked(), out=z(2, 128, 256, dtype=bf16))


@pytest.mark.parametrize("fn", [fq.fp8_quant_act_1x128, fq.fp8_quant_act_1x128_ue8m0, fq.fp8_quant_act_128x1])
def test_activation_quantizer_buffers(fn):
    x = z(200, 256, dtype=bf16)
    with pytest.raises(ValueError, match="K = 200"):
        fn(z(4, 200, dtype=bf16))
    with pytest.raises(ValueError, match="q holds 100"):
        fn(x, q=z(100))
    with pytest.raises(ValueError, match="s holds 7"):
        fn(x, s=z(7, dtype=f32))
    with pytest.raises(ValueError, match="x: expected"):
        fn(z(2, 4, 256, dtype=bf16))
    with pytest.raises(ValueError, match="CUDA tensor"):
        fn(x)


def test_token_axis_scale_count_rounds_rows_up():
    # 200 tokens make two 128-token groups: the scales hold 2 x K floats
    with pytest.raises(ValueError, match="s holds 256 elements, the call needs 512"):
        fq.fp8_quant_act_128x1(z(200, 256, dtype=bf16), s=z(256, dtype=f32))


@pytest.mark.parametrize("fn", [fq.fp8_quant_w_128x128, fq.fp8_quant_w_128x128_ue8m0])
def test_weight_quantizer_buffers(fn):
    w = z(2, 256, 384, dtype=bf16)
    with pytest.raises(ValueError, match="N = 200"):
        fn(z(200, 256, dtype=bf16))
    with pytest.raises(ValueError, match="s holds 6 elements, the call needs 12"):
        fn(w, s=z(6, dtype=f32))              # one batch entry's scales for two
    with pytest.raises(ValueError, match="q holds"):
        fn(w, q=z(256, 384))
    with pytest.raises(ValueError, match="CUDA tensor"):
        fn(w)


def test_transpose_buffers():
    q, s = z(2, 256, 384), z(2, 2, 3, dtype=f32)
    with pytest.raises(ValueError, match="s holds 6"):
        fq.fp8_transpose_w_128x128(q, s[0])
    with pytest.raises(ValueError, match="qt holds"):
        fq.fp8_transpose_w_128x128(q, s, qt=z(384, 256))
    with pytest.raises(ValueError, match="st holds 5"):
        fq.fp8_transpose_w_128x128(q, s, st=z(5, dtype=f32))
    with pytest.raises(ValueError, match="CUDA tensor"):
        fq.fp8_transpose_w_128x128(q, s)


def test_one_device_for_all_arguments():
    """Tensors on two different GPUs are refused (stand-ins carry the two
    attributes the check reads)."""
    d0 = SimpleNamespace(is_cuda=True, device=torch.device("cuda", 0))
    d1 = SimpleNamespace(is_cuda=True, device=torch.device("cuda", 1))
    assert fq._device_of(a=d0, b=None, c=d0) == torch.device("cuda", 0)
    with pytest.raises(ValueError, match="c is on cuda:1"):
        fq._device_of(a=d0, b=d0, c=d1)


def test_swiglu_quant_buffers():
    c1 = z(2, 128, 512, dtype=bf16)
    with pytest.raises(ValueError, match="not 2 x a multiple"):
        fq.fp8_swiglu_quant_1x128(z(4, 384, dtype=bf16))
    with pytest.raises(ValueError, match="masked_m needs c1"):
        fq.fp8_swiglu_quant_1x128(z(256, 512, dtype=bf16), masked_m=z(2, dtype=i32))
    with pytest.raises(ValueError, match="masked_m holds 3"):
        fq.fp8_swiglu_quant_1x128(c1, masked_m=z(3, dtype=i32))
    with pytest.raises(ValueError, match="qh holds 100"):
        fq.fp8_swiglu_quant_1x128(c1, qh=z(100))
    with pytest.raises(ValueError, match="sh holds 7"):
        fq.fp8_swiglu_quant_1x128(c1, sh=z(7, dtype=f32))
    with pytest.raises(ValueError, match="CUDA tensor"):
        fq.fp8_swiglu_quant_1x128(c1, masked_m=z(2, dtype=i32))
def test_token_contiguous_quantizer_buffers():
    x = z(200, 256, dtype=bf16)
    with pytest.raises(ValueError, match="qt holds 51200 elements, the call needs 131072"):
        fq.fp8_quant_act_128x1_t(x, qt=z(256, 200))       # tokens padded to 512 by default
    with pytest.raises(ValueError, match="qt holds 51200 elements, the call needs 65536"):
        fq.fp8_quant_act_128x1_t(x, qt=z(256, 200), Mp=256)
    with pytest.raises(ValueError, match="s holds 256"):
        fq.fp8_quant_act_128x1_t(x, s=z(256, dtype=f32))
    with pytest.raises(ValueError, match="below the token count"):
        fq.fp8_quant_act_128x1_t(x, Mp=128)
    with pytest.raises(ValueError, match="Mp = 300"):
        fq.fp8_quant_act_128x1_t(x, Mp=300)
    with pytest.raises(ValueError, match="CUDA tensor"):
        fq.fp8_quant_act_128x1_t(x)


def test_wgrad_buffers():
    def args(N=256, K=384, Mp=512):
        return [z(N, Mp), z(Mp // 128, N, dtype=f32), z(K, Mp), z(Mp // 128, K, dtype=f32)]
    a = args()
    a[2] = z(384, 384)
    with pytest.raises(ValueError, match="differ in tokens"):
        fq.fp8_gemm_wgrad(*a)
    a = args()
    a[1] = z(256, 4, dtype=f32).t()
    with pytest.raises(ValueError, match="s_dy must be contiguous"):
        fq.fp8_gemm_wgrad(*a)
    a = args()
    a[3] = z(3, 384, dtype=f32)
    with pytest.raises(ValueError, match="s_x holds 1152"):
        fq.fp8_gemm_wgrad(*a)
    with pytest.raises(ValueError, match="Mp = 256 is not a positive multiple of 512"):
        fq.fp8_gemm_wgrad(z(256, 256), z(2, 256, dtype=f32), z(384, 256), z(2, 384, dtype=f32))
    with pytest.raises(ValueError, match="out holds"):
        fq.fp8_gemm_wgrad(*args(), out=z(384, 256 + 1, dtype=bf16))
    with pytest.raises(ValueError, match="CUDA tensor"):
        fq.fp8_gemm_wgrad(*args())
