"""Python binding of ``libfp8q.so``: fine-grained FP8 quantization and
block-scaled FP8 GEMMs for B200 (sm_100a).

Argument marshalling only.  Every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/fp8q.h``; PyTorch provides the
device memory and the stream.  There is no CPU fallback: if the library is
missing or the device is not sm_100, the calls raise.

Names and semantics match the C entry points:

* :func:`fp8_quant_act_1x128`  -- bf16 [M,K] -> E4M3 [M,K] + f32 scales [M,K/128]
* :func:`fp8_quant_w_128x128`  -- bf16 [N,K] or [G,N,K] -> E4M3 + f32 scales [..,N/128,K/128]
* :func:`fp8_quant_act_128x1`  -- bf16 [M,K] -> E4M3 [M,K] + f32 scales [ceil(M/128),K] (token-axis tiles)
* :func:`fp8_quant_act_1x128_ue8m0`, :func:`fp8_quant_w_128x128_ue8m0` -- the same groups, power-of-two scales
* :func:`fp8_transpose_w_128x128` -- block-quantized W [..,N,K] -> W^T [..,K,N] (codes and block scales)
* :func:`fp8_gemm_blockscaled` -- C = A * B^T (bf16) with per-128-slab promotion
* :func:`fp8_grouped_gemm_contiguous` -- MoE grouped GEMM, contiguous layout
* :func:`fp8_grouped_gemm_masked`     -- MoE grouped GEMM, masked layout
"""
from __future__ import annotations

import ctypes
from pathlib import Path

import torch

__all__ = [
    "fp8_quant_act_1x128", "fp8_quant_w_128x128", "fp8_quant_act_128x1", "fp8_transpose_w_128x128",
    "fp8_quant_act_1x128_ue8m0", "fp8_quant_w_128x128_ue8m0",
    "fp8_gemm_blockscaled", "fp8_grouped_gemm_contiguous",
    "fp8_grouped_gemm_masked", "fp8_gemm_unpromoted_diag", "get_device_error", "set_wait_timeout_ns",
    "selftest_wait_timeout", "launch_count", "status_string", "Fp8qError", "lib", "LIB_PATH", "EXPORTS",
]

LIB_PATH = Path(__file__).resolve().parent / "libfp8q.so"
TILE = 128

OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_CUDA, ERR_TIMEOUT, ERR_UNSUPPORTED = range(7)

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
# name -> (restype, argtypes); mirrors include/fp8q.h
EXPORTS = {
    "fp8_quant_act_1x128": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P]),
    "fp8_quant_w_128x128": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P]),
    "fp8_quant_act_128x1": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P]),
    "fp8_quant_act_1x128_ue8m0": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P]),
    "fp8_quant_w_128x128_ue8m0": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P]),
    "fp8_transpose_w_128x128": (ctypes.c_int, [_P, _P, _I64, _I64, _I64, _P, _P, _P]),
    "fp8_gemm_blockscaled": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "fp8_grouped_gemm_contiguous": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _P]),
    "fp8_grouped_gemm_masked": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _P]),
    "fp8_gemm_unpromoted_diag": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "fp8q_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "fp8q_get_device_error": (ctypes.c_int, [_P]),
    "fp8q_set_wait_timeout_ns": (ctypes.c_int, [ctypes.c_uint64]),
    "fp8q_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_uint64, _P]),
    "fp8q_launch_count": (ctypes.c_uint64, []),
}

_lib = None


class Fp8qError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (what, status_string(status), status))


def lib():
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not LIB_PATH.exists():
            raise ImportError("%s is missing: build it with `python -m fp8_fine_grained_quant_b200.build` "
                              "(or __graft_entry__.build())" % LIB_PATH)
        l = ctypes.CDLL(str(LIB_PATH))
        for name, (res, args) in EXPORTS.items():
            fn = getattr(l, name)
            fn.restype = res
            fn.argtypes = args
        _lib = l
    return _lib


def status_string(status: int) -> str:
    return lib().fp8q_status_string(int(status)).decode()


def _check(rc: int, what: str):
    if rc != OK:
        raise Fp8qError(rc, what)


def _stream(stream, device) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _dev(t: torch.Tensor, name: str, dtypes, ndim=None) -> torch.Tensor:
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if t.dtype not in dtypes:
        raise TypeError("%s: dtype %s not in %s" % (name, t.dtype, dtypes))
    if ndim is not None and t.dim() not in ndim:
        raise ValueError("%s: expected %s dims, got %d" % (name, ndim, t.dim()))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t


_FP8 = (torch.float8_e4m3fn, torch.uint8)
_BF16 = (torch.bfloat16,)
_F32 = (torch.float32,)
_I32 = (torch.int32,)


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def fp8_quant_act_1x128(x: torch.Tensor, q: torch.Tensor | None = None, s: torch.Tensor | None = None, stream=None,
                        _entry: str = "fp8_quant_act_1x128"):
    """Online 1x128 activation quantization.  Returns (q [M,K] float8_e4m3fn, s [M,K/128] f32)."""
    _dev(x, "x", _BF16, (2,))
    M, K = x.shape
    if q is None:
        q = torch.empty((M, K), dtype=torch.float8_e4m3fn, device=x.device)
    if s is None:
        s = torch.empty((M, K // TILE), dtype=torch.float32, device=x.device)
    _dev(q, "q", _FP8)
    _dev(s, "s", _F32)
    if q.numel() != M * K or s.numel() != M * (K // TILE):
        raise ValueError("output sizes do not match x")
    with torch.cuda.device(x.device):
        _check(getattr(lib(), _entry)(_p(x), M, K, _p(q), _p(s), _stream(stream, x.device)), _entry)
    return q, s


def fp8_quant_w_128x128(w: torch.Tensor, q: torch.Tensor | None = None, s: torch.Tensor | None = None, stream=None,
                        _entry: str = "fp8_quant_w_128x128"):
    """Online 128x128 weight quantization of [N,K] or [G,N,K] bf16."""
    _dev(w, "w", _BF16, (2, 3))
    G, N, K = (1,) + tuple(w.shape) if w.dim() == 2 else tuple(w.shape)
    lead = tuple(w.shape[:-2])
    if q is None:
        q = torch.empty(tuple(w.shape), dtype=torch.float8_e4m3fn, device=w.device)
    if s is None:
        s = torch.empty(lead + (N // TILE, K // TILE), dtype=torch.float32, device=w.device)
    _dev(q, "q", _FP8)
    _dev(s, "s", _F32)
    if q.numel() != G * N * K or s.numel() != G * (N // TILE) * (K // TILE):
        raise ValueError("output sizes do not match w")
    with torch.cuda.device(w.device):
        _check(getattr(lib(), _entry)(_p(w), G, N, K, _p(q), _p(s), _stream(stream, w.device)), _entry)
    return q, s


def fp8_quant_act_1x128_ue8m0(x, q=None, s=None, stream=None):
    """1x128 activation quantization with power-of-two (UE8M0) scales."""
    return fp8_quant_act_1x128(x, q, s, stream, _entry="fp8_quant_act_1x128_ue8m0")


def fp8_quant_w_128x128_ue8m0(w, q=None, s=None, stream=None):
    """128x128 weight quantization with power-of-two (UE8M0) scales."""
    return fp8_quant_w_128x128(w, q, s, stream, _entry="fp8_quant_w_128x128_ue8m0")


def fp8_quant_act_128x1(x: torch.Tensor, q: torch.Tensor | None = None, s: torch.Tensor | None = None, stream=None):
    """Token-axis (128x1) quantization.  Returns (q [M,K] float8_e4m3fn, s [ceil(M/128),K] f32)."""
    _dev(x, "x", _BF16, (2,))
    M, K = x.shape
    nmb = (M + TILE - 1) // TILE
    if q is None:
        q = torch.empty((M, K), dtype=torch.float8_e4m3fn, device=x.device)
    if s is None:
        s = torch.empty((nmb, K), dtype=torch.float32, device=x.device)
    _dev(q, "q", _FP8)
    _dev(s, "s", _F32)
    if q.numel() != M * K or s.numel() != nmb * K:
        raise ValueError("output sizes do not match x")
    with torch.cuda.device(x.device):
        _check(lib().fp8_quant_act_128x1(_p(x), M, K, _p(q), _p(s), _stream(stream, x.device)), "fp8_quant_act_128x1")
    return q, s


def fp8_transpose_w_128x128(q: torch.Tensor, s: torch.Tensor, qt: torch.Tensor | None = None,
                            st: torch.Tensor | None = None, stream=None):
    """Block-quantized W [N,K] or [G,N,K] (codes + [..,N/128,K/128] scales) -> W^T codes [..,K,N] and
    scales [..,K/128,N/128].  With them, fp8_gemm_blockscaled(q_dy, s_dy, qt, st) is dX = dY W."""
    _dev(q, "q", _FP8, (2, 3))
    _dev(s, "s", _F32)
    G, N, K = (1,) + tuple(q.shape) if q.dim() == 2 else tuple(q.shape)
    lead = tuple(q.shape[:-2])
    if s.numel() != G * (N // TILE) * (K // TILE):
        raise ValueError("scale size does not match q")
    if qt is None:
        qt = torch.empty(lead + (K, N), dtype=torch.float8_e4m3fn, device=q.device)
    if st is None:
        st = torch.empty(lead + (K // TILE, N // TILE), dtype=torch.float32, device=q.device)
    _dev(qt, "qt", _FP8)
    _dev(st, "st", _F32)
    if qt.numel() != G * N * K or st.numel() != G * (N // TILE) * (K // TILE):
        raise ValueError("output sizes do not match q")
    with torch.cuda.device(q.device):
        _check(lib().fp8_transpose_w_128x128(_p(q), _p(s), G, N, K, _p(qt), _p(st), _stream(stream, q.device)),
               "fp8_transpose_w_128x128")
    return qt, st


def _gemm_operands(qa, sa, qb, sb):
    _dev(qa, "qa", _FP8)
    _dev(sa, "sa", _F32)
    _dev(qb, "qb", _FP8)
    _dev(sb, "sb", _F32)


def fp8_gemm_blockscaled(qa, sa, qb, sb, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """C[M,N] (bf16) = A * B^T from 1x128-quantized A and 128x128-quantized B."""
    _gemm_operands(qa, sa, qb, sb)
    M, K = qa.shape
    N = qb.shape[0]
    if tuple(qb.shape) != (N, K) or sa.numel() != M * (K // TILE) or sb.numel() != (N // TILE) * (K // TILE):
        raise ValueError("operand shapes do not agree")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=qa.device)
    _dev(out, "out", _BF16)
    if out.numel() != M * N:
        raise ValueError("out must hold M*N elements")
    with torch.cuda.device(qa.device):
        _check(lib().fp8_gemm_blockscaled(_p(qa), _p(sa), _p(qb), _p(sb), _p(out), M, N, K,
                                          _stream(stream, qa.device)), "fp8_gemm_blockscaled")
    return out


def fp8_gemm_unpromoted_diag(qa, sa, qb, sb, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Diagnostic: all of K accumulated in the tensor cores, scaled once (per-tensor scales only)."""
    _gemm_operands(qa, sa, qb, sb)
    M, K = qa.shape
    N = qb.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=qa.device)
    _dev(out, "out", _BF16)
    with torch.cuda.device(qa.device):
        _check(lib().fp8_gemm_unpromoted_diag(_p(qa), _p(sa), _p(qb), _p(sb), _p(out), M, N, K,
                                              _stream(stream, qa.device)), "fp8_gemm_unpromoted_diag")
    return out


def fp8_grouped_gemm_contiguous(qa, sa, qb, sb, m_indices, out: torch.Tensor | None = None, stream=None):
    """Contiguous-layout grouped GEMM: C[M_tot,N]; block b uses expert m_indices[b]."""
    _gemm_operands(qa, sa, qb, sb)
    _dev(m_indices, "m_indices", _I32)
    M_tot, K = qa.shape
    E, N, K2 = qb.shape
    if K2 != K or m_indices.numel() != M_tot // TILE:
        raise ValueError("operand shapes do not agree")
    if out is None:
        out = torch.empty((M_tot, N), dtype=torch.bfloat16, device=qa.device)
    _dev(out, "out", _BF16)
    with torch.cuda.device(qa.device):
        _check(lib().fp8_grouped_gemm_contiguous(_p(qa), _p(sa), _p(qb), _p(sb), _p(m_indices), _p(out), M_tot, N, K,
                                                 E, _stream(stream, qa.device)), "fp8_grouped_gemm_contiguous")
    return out


def fp8_grouped_gemm_masked(qa, sa, qb, sb, masked_m, expected_m: int = 0, out: torch.Tensor | None = None,
                            stream=None):
    """Masked-layout grouped GEMM: C[E,cap,N]; rows >= masked_m[e] are left unwritten."""
    _gemm_operands(qa, sa, qb, sb)
    _dev(masked_m, "masked_m", _I32)
    E, cap, K = qa.shape
    E2, N, K2 = qb.shape
    if E2 != E or K2 != K or masked_m.numel() != E:
        raise ValueError("operand shapes do not agree")
    if out is None:
        out = torch.empty((E, cap, N), dtype=torch.bfloat16, device=qa.device)
    _dev(out, "out", _BF16)
    with torch.cuda.device(qa.device):
        _check(lib().fp8_grouped_gemm_masked(_p(qa), _p(sa), _p(qb), _p(sb), _p(masked_m), _p(out), E, cap, N, K,
                                             int(expected_m), _stream(stream, qa.device)), "fp8_grouped_gemm_masked")
    return out


def get_device_error(stream=None, device=None) -> int:
    """Synchronizes the stream and returns (and clears) the device status."""
    device = device if device is not None else torch.cuda.current_device()
    with torch.cuda.device(device):
        return int(lib().fp8q_get_device_error(_stream(stream, device)))


def set_wait_timeout_ns(ns: int) -> None:
    _check(lib().fp8q_set_wait_timeout_ns(int(ns)), "fp8q_set_wait_timeout_ns")


def selftest_wait_timeout(ns: int, stream=None, device=None) -> None:
    device = device if device is not None else torch.cuda.current_device()
    with torch.cuda.device(device):
        _check(lib().fp8q_selftest_wait_timeout(int(ns), _stream(stream, device)), "fp8q_selftest_wait_timeout")


def launch_count() -> int:
    return int(lib().fp8q_launch_count())
