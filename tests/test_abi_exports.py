"""The C-ABI library loads on a machine without a GPU, exports every symbol the
header declares, and rejects bad arguments before touching the device.

No call here reaches CUDA: every argument set below fails host-side
validation (shape, NULL or alignment), which the library checks first.
"""
import ctypes
import re
from pathlib import Path

import pytest
import torch

import fp8_fine_grained_quant_b200 as fq

ROOT = Path(__file__).resolve().parents[1]
HEADER = ROOT / "include" / "fp8q.h"


def declared_functions():
    text = HEADER.read_text()
    return re.findall(r"^FP8Q_API\s+[\w\s\*]+?\b(\w+)\s*\(", text, flags=re.M)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    for required in ("fp8_quant_act_1x128", "fp8_quant_w_128x128", "fp8_gemm_blockscaled",
                     "fp8_grouped_gemm_contiguous", "fp8_grouped_gemm_masked", "fp8q_status_string",
                     "fp8q_get_device_error"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = fq.lib()
    raw = ctypes.CDLL(str(fq.LIB_PATH))
    for name in declared_functions():
        assert hasattr(raw, name), name
        assert name in fq.EXPORTS, "binding lacks %s" % name
        assert hasattr(lib, name)
    assert set(fq.EXPORTS) == set(declared_functions())


def test_internal_symbols_hidden():
    out = ctypes.CDLL(str(fq.LIB_PATH))
    with pytest.raises(AttributeError):
        out.make_operand_map  # noqa: B018  (C++ internals are not exported)


def test_status_strings():
    assert fq.status_string(0) == "ok"
    for s in range(1, 7):
        assert fq.status_string(s) not in ("ok", "unknown status")
    assert fq.status_string(99) == "unknown status"


A16 = 0x10000  # a 256-byte aligned fake address; never dereferenced
A16_ONLY = 0x10010  # 16-byte but not 32-byte aligned
A4 = 0x10004   # 4-byte aligned only
A1 = 0x10001
BIG_ = 1 << 31


def _call(name, *args):
    return getattr(fq.lib(), name)(*args)


@pytest.mark.parametrize("args,expect", [
    ((A16, 4, 100, A16, A16, None), fq.ERR_SHAPE),     # K not a multiple of 128
    ((A16, -1, 128, A16, A16, None), fq.ERR_SHAPE),
    ((A16, 0, 128, A16, A16, None), fq.OK),            # empty: no-op
    ((A16, 4, 0, A16, A16, None), fq.OK),
    ((None, 4, 128, A16, A16, None), fq.ERR_NULL),
    ((A16, 4, 128, None, A16, None), fq.ERR_NULL),
    ((A4, 4, 128, A16, A16, None), fq.ERR_ALIGN),
    ((A16_ONLY, 4, 128, A16, A16, None), fq.ERR_ALIGN),  # bf16 input: 32 bytes
    ((A16, 4, 128, A4, A16, None), fq.ERR_ALIGN),
    ((A16, 4, 128, A16, A1, None), fq.ERR_ALIGN),
])
def test_quant_act_validation(args, expect):
    assert _call("fp8_quant_act_1x128", *args) == expect


@pytest.mark.parametrize("args,expect", [
    ((A16, 1, 100, 128, A16, A16, None), fq.ERR_SHAPE),
    ((A16, 1, 128, 129, A16, A16, None), fq.ERR_SHAPE),
    ((A16, 0, 128, 128, A16, A16, None), fq.OK),
    ((None, 1, 128, 128, A16, A16, None), fq.ERR_NULL),
    ((A16, 2, 128, 128, A16, A1, None), fq.ERR_ALIGN),
    ((A16_ONLY, 1, 128, 128, A16, A16, None), fq.ERR_ALIGN),  # bf16 input: 32 bytes
])
def test_quant_w_validation(args, expect):
    assert _call("fp8_quant_w_128x128", *args) == expect


@pytest.mark.parametrize("args,expect", [
    ((A16, 4, 100, A16, A16, A16, 1, 128, 128, A16, A16, None), fq.ERR_SHAPE),   # activation K
    ((A16, 4, 128, A16, A16, A16, 1, 100, 128, A16, A16, None), fq.ERR_SHAPE),   # weight N
    ((A16, 4, 128, A16, A16, A16, 1, 128, 100, A16, A16, None), fq.ERR_SHAPE),   # weight K
    ((A16, BIG_, 128, A16, A16, A16, 1, 128, 128, A16, A16, None), fq.ERR_SHAPE),
    ((A16, 4, 128, A16, A16, A16, 1 << 24, 1 << 8, 128, A16, A16, None), fq.ERR_SHAPE),  # G*N = 2^32
    ((None, 4, 128, A16, A16, A16, 1, 128, 128, A16, A16, None), fq.ERR_NULL),
    ((A16, 4, 128, A16, A16, None, 1, 128, 128, A16, A16, None), fq.ERR_NULL),
    ((A16, 4, 128, A16, A16, A16, 1, 128, 128, A16, None, None), fq.ERR_NULL),
    ((A16_ONLY, 4, 128, A16, A16, A16, 1, 128, 128, A16, A16, None), fq.ERR_ALIGN),
    ((A16, 4, 128, A16, A16, A16_ONLY, 1, 128, 128, A16, A16, None), fq.ERR_ALIGN),
    ((A16, 4, 128, A16, A1, A16, 1, 128, 128, A16, A16, None), fq.ERR_ALIGN),
    ((A16, 0, 128, A16, A16, A16, 0, 128, 128, A16, A16, None), fq.OK),           # both empty
    ((None, 0, 128, None, None, None, 0, 128, 128, None, None, None), fq.OK),     # empty parts need no pointers
])
def test_quant_act_w_validation(args, expect):
    """The fused two-operand quantizer checks both operands' shapes, pointers
    and alignment before anything is launched."""
    assert _call("fp8_quant_act_w", *args) == expect


@pytest.mark.parametrize("name", ["fp8_gemm_blockscaled", "fp8_gemm_unpromoted_diag"])
@pytest.mark.parametrize("mnk,ptrs,expect", [
    ((128, 256, 100), (A16,) * 5, fq.ERR_SHAPE),
    ((128, 200, 128), (A16,) * 5, fq.ERR_SHAPE),
    ((128, 256, 0), (A16,) * 5, fq.ERR_SHAPE),   # K >= 128 required
    ((-1, 256, 128), (A16,) * 5, fq.ERR_SHAPE),
    ((0, 256, 128), (A16,) * 5, fq.OK),
    ((128, 0, 128), (A16,) * 5, fq.OK),
    ((128, 256, 128), (None, A16, A16, A16, A16), fq.ERR_NULL),
    ((128, 256, 128), (A16, A16, A16, A16, None), fq.ERR_NULL),
    ((128, 256, 128), (A4, A16, A16, A16, A16), fq.ERR_ALIGN),
    ((128, 256, 128), (A16, A1, A16, A16, A16), fq.ERR_ALIGN),
    ((128, 256, 128), (A16, A16, A16, A16, A4), fq.ERR_ALIGN),
])
def test_gemm_validation(name, mnk, ptrs, expect):
    assert _call(name, *ptrs, *mnk, None) == expect


@pytest.mark.parametrize("args,expect", [
    ((A16, A16, A16, A16, A16, A16, 200, 256, 128, 4), fq.ERR_SHAPE),   # M_tot % 128
    ((A16, A16, A16, A16, A16, A16, 256, 256, 100, 4), fq.ERR_SHAPE),
    ((A16, A16, A16, A16, A16, A16, 0, 256, 128, 4), fq.OK),
    ((A16, A16, A16, A16, A16, A16, 256, 256, 128, 0), fq.OK),          # no expert: nothing written
    ((A16, A16, A16, A16, None, A16, 256, 256, 128, 4), fq.ERR_NULL),
    ((A16, A16, A16, A16, A1, A16, 256, 256, 128, 4), fq.ERR_ALIGN),
])
def test_contiguous_validation(args, expect):
    assert _call("fp8_grouped_gemm_contiguous", *args, None) == expect


@pytest.mark.parametrize("args,expect", [
    ((A16, A16, A16, A16, A16, A16, 4, 200, 256, 128, 0), fq.ERR_SHAPE),  # cap % 128
    ((A16, A16, A16, A16, A16, A16, 2000, 128, 256, 128, 0), fq.ERR_SHAPE),  # E > 1024
    ((A16, A16, A16, A16, A16, A16, 4, 128, 256, 128, -1), fq.ERR_SHAPE),
    ((A16, A16, A16, A16, A16, A16, 0, 128, 256, 128, 0), fq.OK),
    ((A16, A16, A16, A16, None, A16, 4, 128, 256, 128, 0), fq.ERR_NULL),
    ((A16, A16, A16, A16, A1, A16, 4, 128, 256, 128, 0), fq.ERR_ALIGN),
])
def test_masked_validation(args, expect):
    assert _call("fp8_grouped_gemm_masked", *args, None) == expect


def test_binding_rejects_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        fq.fp8_quant_act_1x128(torch.zeros(4, 128, dtype=torch.bfloat16))


@pytest.mark.parametrize("args,expect", [
    ((A16, 4, 100, A16, A16, None), fq.ERR_SHAPE),    # K not a multiple of 128
    ((A16, -1, 128, A16, A16, None), fq.ERR_SHAPE),
    ((A16, 0, 128, A16, A16, None), fq.OK),
    ((None, 4, 128, A16, A16, None), fq.ERR_NULL),
    ((A16, 4, 128, A16, A4, None), fq.ERR_ALIGN),     # scales written as 16-byte vectors
])
def test_quant_act_128x1_validation(args, expect):
    assert _call("fp8_quant_act_128x1", *args) == expect


@pytest.mark.parametrize("args,expect", [
    ((A16, A16, 1, 100, 128, A16, A16, None), fq.ERR_SHAPE),
    ((A16, A16, 1, 128, 0, A16, A16, None), fq.OK),
    ((A16, None, 1, 128, 128, A16, A16, None), fq.ERR_NULL),
    ((A16, A16, 1, 128, 128, A4, A16, None), fq.ERR_ALIGN),
])
def test_transpose_w_validation(args, expect):
    assert _call("fp8_transpose_w_128x128", *args) == expect


@pytest.mark.parametrize("name,args,expect", [
    ("fp8_quant_act_1x128_ue8m0", (A16, 4, 100, A16, A16, None), fq.ERR_SHAPE),
    ("fp8_quant_act_1x128_ue8m0", (A16_ONLY, 4, 128, A16, A16, None), fq.ERR_ALIGN),
    ("fp8_quant_act_1x128_ue8m0", (A16, 0, 128, A16, A16, None), fq.OK),
    ("fp8_quant_w_128x128_ue8m0", (A16, 1, 100, 128, A16, A16, None), fq.ERR_SHAPE),
    ("fp8_quant_w_128x128_ue8m0", (None, 1, 128, 128, A16, A16, None), fq.ERR_NULL),
])
def test_ue8m0_quant_validation(name, args, expect):
    assert _call(name, *args) == expect


@pytest.mark.parametrize("call", [
    lambda: fq.fp8_quant_act_1x128(torch.zeros((4, 128), dtype=torch.bfloat16)),
    lambda: fq.fp8_quant_w_128x128(torch.zeros((128, 128), dtype=torch.bfloat16)),
    lambda: fq.fp8_quant_act_128x1(torch.zeros((4, 128), dtype=torch.bfloat16)),
    lambda: fq.fp8_quant_act_1x128_ue8m0(torch.zeros((4, 128), dtype=torch.bfloat16)),
    lambda: fq.fp8_gemm_blockscaled(torch.zeros((4, 128), dtype=torch.uint8), torch.ones((4, 1)),
                                    torch.zeros((128, 128), dtype=torch.uint8), torch.ones((1, 1))),
    lambda: fq.fp8_transpose_w_128x128(torch.zeros((128, 128), dtype=torch.uint8), torch.ones((1, 1))),
])
def test_no_cpu_fallback(call):
    """Host tensors are refused before anything runs: there is no CPU path."""
    with pytest.raises(ValueError, match="CUDA tensor"):
        call()


BIG = 1 << 31


@pytest.mark.parametrize("name,args", [
    ("fp8_quant_act_1x128", (A16, BIG, 128, A16, A16, None)),
    ("fp8_quant_act_1x128", (A16, 4, BIG, A16, A16, None)),
    ("fp8_quant_act_1x128_ue8m0", (A16, BIG, 128, A16, A16, None)),
    ("fp8_quant_w_128x128", (A16, 1 << 24, 1 << 8, 128, A16, A16, None)),   # G*N = 2^32 stacked rows
    ("fp8_quant_w_128x128", (A16, 1, 128, BIG, A16, A16, None)),
    ("fp8_quant_w_128x128_ue8m0", (A16, BIG, 128, 128, A16, A16, None)),
    ("fp8_quant_act_128x1", (A16, BIG, 128, A16, A16, None)),
    ("fp8_transpose_w_128x128", (A16, A16, 1 << 24, 1 << 8, 128, A16, A16, None)),
])
def test_sizes_beyond_the_limits_are_refused(name, args):
    """Row and column counts of 2^31 or more (and stacked counts that reach
    it) are refused before any index arithmetic could overflow."""
    assert _call(name, *args) == fq.ERR_SHAPE


@pytest.mark.parametrize("args,expect", [
    ((A16, 4, 100, None, 0, A16, A16, None), fq.ERR_SHAPE),      # inter not a multiple of 128
    ((A16, -1, 128, None, 0, A16, A16, None), fq.ERR_SHAPE),
    ((A16, 300, 128, A16, 256, A16, A16, None), fq.ERR_SHAPE),   # masked: cap does not divide rows
    ((A16, 256, 128, A16, 0, A16, A16, None), fq.ERR_SHAPE),
    ((A16, 0, 128, None, 0, A16, A16, None), fq.OK),
    ((None, 4, 128, None, 0, A16, A16, None), fq.ERR_NULL),
    ((A16_ONLY, 4, 128, None, 0, A16, A16, None), fq.ERR_ALIGN),  # bf16 input: 32 bytes
    ((A16, 256, 128, A1, 128, A16, A16, None), fq.ERR_ALIGN),
])
def test_swiglu_quant_validation(args, expect):
    assert _call("fp8_swiglu_quant_1x128", *args) == expect
@pytest.mark.parametrize("args,expect", [
    ((A16, 4, 100, 128, A16, A16, None), fq.ERR_SHAPE),
    ((A16, -1, 128, 128, A16, A16, None), fq.ERR_SHAPE),
    ((A16, 200, 128, 128, A16, A16, None), fq.ERR_SHAPE),   # padded count below the tokens
    ((A16, 4, 128, 200, A16, A16, None), fq.ERR_SHAPE),     # padded count not a multiple of 128
    ((A16, 0, 128, 0, A16, A16, None), fq.OK),
    ((None, 4, 128, 128, A16, A16, None), fq.ERR_NULL),
    ((A16, 4, 128, 128, A16_ONLY + 4, A16, None), fq.ERR_ALIGN),
    ((A16, 4, 128, 512, A16, A4, None), fq.ERR_ALIGN),
])
def test_quant_act_128x1_t_validation(args, expect):
    assert _call("fp8_quant_act_128x1_t", *args) == expect


@pytest.mark.parametrize("nkm,ptrs,expect", [
    ((256, 256, 100), (A16,) * 5, fq.ERR_SHAPE),    # tokens not a multiple of 128
    ((256, 256, 384), (A16,) * 5, fq.ERR_SHAPE),    # nor of a group of four slabs
    ((256, 256, 0), (A16,) * 5, fq.ERR_SHAPE),      # at least one group
    ((200, 256, 512), (A16,) * 5, fq.ERR_SHAPE),
    ((256, 200, 512), (A16,) * 5, fq.ERR_SHAPE),
    ((0, 256, 512), (A16,) * 5, fq.OK),
    ((256, 256, 512), (A16, None, A16, A16, A16), fq.ERR_NULL),
    ((256, 256, 512), (A16, A4, A16, A16, A16), fq.ERR_ALIGN),   # row scales are staged in 16-byte boxes
    ((256, 256, 512), (A16, A16, A16, A16, A1), fq.ERR_ALIGN),
])
def test_wgrad_validation(nkm, ptrs, expect):
    assert _call("fp8_gemm_wgrad", *ptrs, *nkm, None) == expect


@pytest.mark.parametrize("name,args,expect", [
    ("fp8_mx_scales_act", (A16, 4, 100, A16, None), fq.ERR_SHAPE),
    ("fp8_mx_scales_act", (A16, 0, 128, A16, None), fq.OK),
    ("fp8_mx_scales_act", (None, 4, 128, A16, None), fq.ERR_NULL),
    ("fp8_mx_scales_act", (A16, 4, 128, A4, None), fq.ERR_ALIGN),
    ("fp8_mx_scales_w", (A16, 1, 100, 128, A16, None), fq.ERR_SHAPE),
    ("fp8_mx_scales_w", (A16, 1, 128, 128, A1, None), fq.ERR_ALIGN),
    ("fp8_gemm_mx", (A16, A16, A16, A16, A16, 128, 256, 100, None), fq.ERR_SHAPE),
    ("fp8_gemm_mx", (A16, A16, A16, A16, A16, 0, 256, 128, None), fq.OK),
    ("fp8_gemm_mx", (A16, None, A16, A16, A16, 128, 256, 128, None), fq.ERR_NULL),
    ("fp8_gemm_mx", (A16, A4, A16, A16, A16, 128, 256, 128, None), fq.ERR_ALIGN),   # bulk-copied atoms
])
def test_mx_validation(name, args, expect):
    assert _call(name, *args) == expect


@pytest.mark.parametrize("name,args,expect", [
    ("fp8_grouped_gemm_mx_contiguous", (A16, A16, A16, A16, A16, A16, 200, 256, 128, 4, None), fq.ERR_SHAPE),
    ("fp8_grouped_gemm_mx_contiguous", (A16, A16, A16, A16, None, A16, 256, 256, 128, 4, None), fq.ERR_NULL),
    ("fp8_grouped_gemm_mx_contiguous", (A16, A4, A16, A16, A16, A16, 256, 256, 128, 4, None), fq.ERR_ALIGN),
    ("fp8_grouped_gemm_mx_masked", (A16, A16, A16, A16, A16, A16, 4, 200, 256, 128, None), fq.ERR_SHAPE),
    ("fp8_grouped_gemm_mx_masked", (A16, A16, A16, A16, A16, A16, 0, 128, 256, 128, None), fq.OK),
    ("fp8_grouped_gemm_mx_masked", (A16, A16, A16, A16, A1, A16, 4, 128, 256, 128, None), fq.ERR_ALIGN),
])
def test_grouped_mx_validation(name, args, expect):
    assert _call(name, *args) == expect
