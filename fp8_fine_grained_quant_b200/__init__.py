"""Python binding of ``libfp8q.so``: fine-grained FP8 quantization and
block-scaled FP8 GEMMs for B200 (sm_100a).

Argument marshalling only.  Every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/fp8q.h``; PyTorch provides the
device memory and the stream.  There is no CPU fallback: if the library is
missing or the device is not sm_100, the calls raise.

Names and semantics match the C entry points:

* :func:`fp8_quant_act_1x128`  -- bf16 [M,K] -> E4M3 [M,K] + f32 scales [M,K/128]
* :func:`fp8_quant_w_128x128`  -- bf16 [N,K] or [G,N,K] -> E4M3 + f32 scales [..,N/128,K/128]
* :func:`fp8_quant_act_w`      -- both of the above in one launch (the two operands of one GEMM)
* :func:`fp8_quant_act_128x1`  -- bf16 [M,K] -> E4M3 [M,K] + f32 scales [ceil(M/128),K] (token-axis tiles)
* :func:`fp8_quant_act_128x1_t` -- the same groups, codes token-contiguous: E4M3 [K,Mp] (tokens padded to Mp)
* :func:`fp8_quant_act_1x128_ue8m0`, :func:`fp8_quant_w_128x128_ue8m0` -- the same groups, power-of-two scales
* :func:`fp8_transpose_w_128x128` -- block-quantized W [..,N,K] -> W^T [..,K,N] (codes and block scales)
* :func:`fp8_swiglu_quant_1x128` -- GEMM1 output [.., 2I] bf16 -> SwiGLU -> 1x128 E4M3 [.., I] + scales
* :func:`fp8_mx_scales_act`, :func:`fp8_mx_scales_w`, :func:`fp8_gemm_mx` -- power-of-two scales applied by
  the tensor cores (E8M0 scale atoms, no CUDA-core promotion)
* :func:`fp8_gemm_blockscaled` -- C = A * B^T (bf16) with per-128-slab promotion
* :func:`fp8_grouped_gemm_contiguous` -- MoE grouped GEMM, contiguous layout
* :func:`fp8_grouped_gemm_masked`     -- MoE grouped GEMM, masked layout
* :func:`fp8_gemm_wgrad`       -- dW [N,K] = dY^T X over tokens, both operands token-axis quantized
"""
from __future__ import annotations

import ctypes
from pathlib import Path

import torch

__all__ = [
    "fp8_quant_act_1x128", "fp8_quant_w_128x128", "fp8_quant_act_w", "fp8_quant_act_128x1", "fp8_quant_act_128x1_t",
    "fp8_transpose_w_128x128", "fp8_gemm_wgrad", "fp8_swiglu_quant_1x128",
    "fp8_quant_act_1x128_ue8m0", "fp8_quant_w_128x128_ue8m0",
    "fp8_gemm_blockscaled", "fp8_grouped_gemm_contiguous",
    "fp8_grouped_gemm_masked", "fp8_gemm_unpromoted_diag", "fp8_mx_scales_act", "fp8_mx_scales_w", "fp8_gemm_mx",
    "fp8_grouped_gemm_mx_contiguous", "fp8_grouped_gemm_mx_masked", "get_device_error", "set_wait_timeout_ns",
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
    "fp8_quant_act_w": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P, _I64, _I64, _I64, _P, _P, _P]),
    "fp8_quant_act_128x1": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P]),
    "fp8_quant_act_128x1_t": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P]),
    "fp8_quant_act_1x128_ue8m0": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P]),
    "fp8_quant_w_128x128_ue8m0": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P]),
    "fp8_transpose_w_128x128": (ctypes.c_int, [_P, _P, _I64, _I64, _I64, _P, _P, _P]),
    "fp8_swiglu_quant_1x128": (ctypes.c_int, [_P, _I64, _I64, _P, _I64, _P, _P, _P]),
    "fp8_gemm_blockscaled": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "fp8_grouped_gemm_contiguous": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _P]),
    "fp8_grouped_gemm_masked": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _P]),
    "fp8_gemm_unpromoted_diag": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "fp8_mx_scales_act": (ctypes.c_int, [_P, _I64, _I64, _P, _P]),
    "fp8_mx_scales_w": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P]),
    "fp8_gemm_mx": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "fp8_grouped_gemm_mx_contiguous": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _P]),
    "fp8_grouped_gemm_mx_masked": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _P]),
    "fp8_gemm_wgrad": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P]),
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


def _tensor(t, name: str, dtypes, ndim=None):
    """Type, dtype, rank and layout of one argument (the device is checked
    once for all arguments by :func:`_device_of`)."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if t.dtype not in dtypes:
        raise TypeError("%s: dtype %s not in %s" % (name, t.dtype, dtypes))
    if ndim is not None and t.dim() not in ndim:
        raise ValueError("%s: expected %s dims, got %d" % (name, ndim, t.dim()))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t


def _numel(t, n: int, name: str):
    """A caller-supplied buffer must hold exactly the elements the call reads
    or writes: the C library trusts the sizes it is given."""
    if t is not None and t.numel() != n:
        raise ValueError("%s holds %d elements, the call needs %d" % (name, t.numel(), n))


def _device_of(**tensors) -> torch.device:
    """All tensors are CUDA tensors on one device (there is no CPU path)."""
    dev = None
    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("%s must be a CUDA tensor" % name)
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError("%s is on %s, the other arguments on %s" % (name, t.device, dev))
    return dev


_FP8 = (torch.float8_e4m3fn, torch.uint8)
_BF16 = (torch.bfloat16,)
_F32 = (torch.float32,)
_I32 = (torch.int32,)


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _multiple(v: int, name: str):
    if v % TILE:
        raise ValueError("%s = %d is not a multiple of %d" % (name, v, TILE))


def fp8_quant_act_1x128(x: torch.Tensor, q: torch.Tensor | None = None, s: torch.Tensor | None = None, stream=None,
                        _entry: str = "fp8_quant_act_1x128"):
    """Online 1x128 activation quantization.  Returns (q [M,K] float8_e4m3fn, s [M,K/128] f32)."""
    _tensor(x, "x", _BF16, (2,))
    M, K = x.shape
    _multiple(K, "K")
    _tensor(q, "q", _FP8)
    _tensor(s, "s", _F32)
    _numel(q, M * K, "q")
    _numel(s, M * (K // TILE), "s")
    dev = _device_of(x=x, q=q, s=s)
    if q is None:
        q = torch.empty((M, K), dtype=torch.float8_e4m3fn, device=dev)
    if s is None:
        s = torch.empty((M, K // TILE), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _check(getattr(lib(), _entry)(_p(x), M, K, _p(q), _p(s), _stream(stream, dev)), _entry)
    return q, s


def fp8_quant_w_128x128(w: torch.Tensor, q: torch.Tensor | None = None, s: torch.Tensor | None = None, stream=None,
                        _entry: str = "fp8_quant_w_128x128"):
    """Online 128x128 weight quantization of [N,K] or [G,N,K] bf16."""
    _tensor(w, "w", _BF16, (2, 3))
    G, N, K = (1,) + tuple(w.shape) if w.dim() == 2 else tuple(w.shape)
    _multiple(N, "N")
    _multiple(K, "K")
    lead = tuple(w.shape[:-2])
    _tensor(q, "q", _FP8)
    _tensor(s, "s", _F32)
    _numel(q, G * N * K, "q")
    _numel(s, G * (N // TILE) * (K // TILE), "s")
    dev = _device_of(w=w, q=q, s=s)
    if q is None:
        q = torch.empty(tuple(w.shape), dtype=torch.float8_e4m3fn, device=dev)
    if s is None:
        s = torch.empty(lead + (N // TILE, K // TILE), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _check(getattr(lib(), _entry)(_p(w), G, N, K, _p(q), _p(s), _stream(stream, dev)), _entry)
    return q, s


def fp8_quant_act_w(x: torch.Tensor, w: torch.Tensor, qa: torch.Tensor | None = None, sa: torch.Tensor | None = None,
                    qw: torch.Tensor | None = None, sw: torch.Tensor | None = None, stream=None):
    """Both GEMM operands in one launch: returns ((qa, sa), (qw, sw)), exactly what
    :func:`fp8_quant_act_1x128` (x) and :func:`fp8_quant_w_128x128` (w) return."""
    _tensor(x, "x", _BF16, (2,))
    _tensor(w, "w", _BF16, (2, 3))
    M, K = x.shape
    _multiple(K, "K")
    G, N, Kw = (1,) + tuple(w.shape) if w.dim() == 2 else tuple(w.shape)
    _multiple(N, "N")
    _multiple(Kw, "K of w")
    for t, name, dt in ((qa, "qa", _FP8), (sa, "sa", _F32), (qw, "qw", _FP8), (sw, "sw", _F32)):
        _tensor(t, name, dt)
    _numel(qa, M * K, "qa")
    _numel(sa, M * (K // TILE), "sa")
    _numel(qw, G * N * Kw, "qw")
    _numel(sw, G * (N // TILE) * (Kw // TILE), "sw")
    dev = _device_of(x=x, w=w, qa=qa, sa=sa, qw=qw, sw=sw)
    if qa is None:
        qa = torch.empty((M, K), dtype=torch.float8_e4m3fn, device=dev)
    if sa is None:
        sa = torch.empty((M, K // TILE), dtype=torch.float32, device=dev)
    if qw is None:
        qw = torch.empty(tuple(w.shape), dtype=torch.float8_e4m3fn, device=dev)
    if sw is None:
        sw = torch.empty(tuple(w.shape[:-2]) + (N // TILE, Kw // TILE), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _check(lib().fp8_quant_act_w(_p(x), M, K, _p(qa), _p(sa), _p(w), G, N, Kw, _p(qw), _p(sw),
                                     _stream(stream, dev)), "fp8_quant_act_w")
    return (qa, sa), (qw, sw)


def fp8_quant_act_1x128_ue8m0(x, q=None, s=None, stream=None):
    """1x128 activation quantization with power-of-two (UE8M0) scales."""
    return fp8_quant_act_1x128(x, q, s, stream, _entry="fp8_quant_act_1x128_ue8m0")


def fp8_quant_w_128x128_ue8m0(w, q=None, s=None, stream=None):
    """128x128 weight quantization with power-of-two (UE8M0) scales."""
    return fp8_quant_w_128x128(w, q, s, stream, _entry="fp8_quant_w_128x128_ue8m0")


def fp8_quant_act_128x1(x: torch.Tensor, q: torch.Tensor | None = None, s: torch.Tensor | None = None, stream=None):
    """Token-axis (128x1) quantization.  Returns (q [M,K] float8_e4m3fn, s [ceil(M/128),K] f32)."""
    _tensor(x, "x", _BF16, (2,))
    M, K = x.shape
    _multiple(K, "K")
    nmb = (M + TILE - 1) // TILE
    _tensor(q, "q", _FP8)
    _tensor(s, "s", _F32)
    _numel(q, M * K, "q")
    _numel(s, nmb * K, "s")
    dev = _device_of(x=x, q=q, s=s)
    if q is None:
        q = torch.empty((M, K), dtype=torch.float8_e4m3fn, device=dev)
    if s is None:
        s = torch.empty((nmb, K), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _check(lib().fp8_quant_act_128x1(_p(x), M, K, _p(q), _p(s), _stream(stream, dev)), "fp8_quant_act_128x1")
    return q, s


WGRAD_TOKEN_GROUP = 4 * TILE  # fp8_gemm_wgrad contracts over whole groups of four 128-token slabs


def fp8_quant_act_128x1_t(x: torch.Tensor, qt: torch.Tensor | None = None, s: torch.Tensor | None = None,
                          Mp: int | None = None, stream=None):
    """Token-axis (128x1) quantization with token-contiguous codes, the operand layout of
    :func:`fp8_gemm_wgrad`.  Returns (qt [K, Mp] float8_e4m3fn, s [Mp/128, K] f32) for tokens padded
    to Mp (default: M rounded up to 512, what fp8_gemm_wgrad takes); padding tokens get code 0."""
    _tensor(x, "x", _BF16, (2,))
    M, K = x.shape
    _multiple(K, "K")
    if Mp is None:
        Mp = -(-M // WGRAD_TOKEN_GROUP) * WGRAD_TOKEN_GROUP
    _multiple(Mp, "Mp")
    if Mp < M:
        raise ValueError("Mp = %d is below the token count %d" % (Mp, M))
    _tensor(qt, "qt", _FP8)
    _tensor(s, "s", _F32)
    _numel(qt, K * Mp, "qt")
    _numel(s, (Mp // TILE) * K, "s")
    dev = _device_of(x=x, qt=qt, s=s)
    if qt is None:
        qt = torch.empty((K, Mp), dtype=torch.float8_e4m3fn, device=dev)
    if s is None:
        s = torch.empty((Mp // TILE, K), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _check(lib().fp8_quant_act_128x1_t(_p(x), M, K, Mp, _p(qt), _p(s), _stream(stream, dev)),
               "fp8_quant_act_128x1_t")
    return qt, s


def fp8_transpose_w_128x128(q: torch.Tensor, s: torch.Tensor, qt: torch.Tensor | None = None,
                            st: torch.Tensor | None = None, stream=None):
    """Block-quantized W [N,K] or [G,N,K] (codes + [..,N/128,K/128] scales) -> W^T codes [..,K,N] and
    scales [..,K/128,N/128].  With them, fp8_gemm_blockscaled(q_dy, s_dy, qt, st) is dX = dY W."""
    _tensor(q, "q", _FP8, (2, 3))
    _tensor(s, "s", _F32)
    G, N, K = (1,) + tuple(q.shape) if q.dim() == 2 else tuple(q.shape)
    _multiple(N, "N")
    _multiple(K, "K")
    lead = tuple(q.shape[:-2])
    _numel(s, G * (N // TILE) * (K // TILE), "s")
    _tensor(qt, "qt", _FP8)
    _tensor(st, "st", _F32)
    _numel(qt, G * N * K, "qt")
    _numel(st, G * (N // TILE) * (K // TILE), "st")
    dev = _device_of(q=q, s=s, qt=qt, st=st)
    if qt is None:
        qt = torch.empty(lead + (K, N), dtype=torch.float8_e4m3fn, device=dev)
    if st is None:
        st = torch.empty(lead + (K // TILE, N // TILE), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _check(lib().fp8_transpose_w_128x128(_p(q), _p(s), G, N, K, _p(qt), _p(st), _stream(stream, dev)),
               "fp8_transpose_w_128x128")
    return qt, st


def fp8_swiglu_quant_1x128(c1: torch.Tensor, masked_m: torch.Tensor | None = None, qh: torch.Tensor | None = None,
                           sh: torch.Tensor | None = None, stream=None):
    """SwiGLU of GEMM1's [gate | up] output fused with its 1x128 requantization.
    c1 [rows, 2I] or [E, cap, 2I] bf16 -> (qh [.., I] float8_e4m3fn, sh [.., I/128] f32).  With
    masked_m (int32 [E], c1 3-D), rows at or past masked_m[e] are left unwritten."""
    _tensor(c1, "c1", _BF16, (2, 3))
    _tensor(masked_m, "masked_m", _I32)
    if c1.shape[-1] % (2 * TILE):
        raise ValueError("c1's last dim %d is not 2 x a multiple of %d" % (c1.shape[-1], TILE))
    inter = c1.shape[-1] // 2
    lead = tuple(c1.shape[:-1])
    rows = 1
    for d in lead:
        rows *= d
    cap = 0
    if masked_m is not None:
        if c1.dim() != 3:
            raise ValueError("masked_m needs c1 as [E, cap, 2I]")
        cap = c1.shape[1]
        _numel(masked_m, c1.shape[0], "masked_m")
    _tensor(qh, "qh", _FP8)
    _tensor(sh, "sh", _F32)
    _numel(qh, rows * inter, "qh")
    _numel(sh, rows * (inter // TILE), "sh")
    dev = _device_of(c1=c1, masked_m=masked_m, qh=qh, sh=sh)
    if qh is None:
        qh = torch.empty(lead + (inter,), dtype=torch.float8_e4m3fn, device=dev)
    if sh is None:
        sh = torch.empty(lead + (inter // TILE,), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _check(lib().fp8_swiglu_quant_1x128(_p(c1), rows, inter, _p(masked_m), cap, _p(qh), _p(sh),
                                            _stream(stream, dev)), "fp8_swiglu_quant_1x128")
    return qh, sh


def _dense_operands(qa, sa, qb, sb, out):
    """Shapes of C = A * B^T: qa [M,K], sa [M,K/128], qb [N,K], sb [N/128,K/128], out [M,N]."""
    _tensor(qa, "qa", _FP8, (2,))
    _tensor(sa, "sa", _F32)
    _tensor(qb, "qb", _FP8, (2,))
    _tensor(sb, "sb", _F32)
    _tensor(out, "out", _BF16)
    M, K = qa.shape
    N = qb.shape[0]
    if qb.shape[1] != K:
        raise ValueError("qa and qb differ in K (%d, %d)" % (K, qb.shape[1]))
    _multiple(N, "N")
    _multiple(K, "K")
    _numel(sa, M * (K // TILE), "sa")
    _numel(sb, (N // TILE) * (K // TILE), "sb")
    _numel(out, M * N, "out")
    return M, N, K, _device_of(qa=qa, sa=sa, qb=qb, sb=sb, out=out)


def fp8_gemm_blockscaled(qa, sa, qb, sb, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """C[M,N] (bf16) = A * B^T from 1x128-quantized A and 128x128-quantized B."""
    M, N, K, dev = _dense_operands(qa, sa, qb, sb, out)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    with torch.cuda.device(dev):
        _check(lib().fp8_gemm_blockscaled(_p(qa), _p(sa), _p(qb), _p(sb), _p(out), M, N, K,
                                          _stream(stream, dev)), "fp8_gemm_blockscaled")
    return out


def fp8_gemm_unpromoted_diag(qa, sa, qb, sb, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Diagnostic: all of K accumulated in the tensor cores, scaled once (per-tensor scales only)."""
    M, N, K, dev = _dense_operands(qa, sa, qb, sb, out)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    with torch.cuda.device(dev):
        _check(lib().fp8_gemm_unpromoted_diag(_p(qa), _p(sa), _p(qb), _p(sb), _p(out), M, N, K,
                                              _stream(stream, dev)), "fp8_gemm_unpromoted_diag")
    return out


def fp8_gemm_wgrad(q_dy_t, s_dy, q_x_t, s_x, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """dW [N, K] (bf16) = dY^T X from the token-contiguous quantizations of dY [M, N] and
    X [M, K] (:func:`fp8_quant_act_128x1_t`): q_dy_t [N, Mp], s_dy [Mp/128, N], q_x_t [K, Mp],
    s_x [Mp/128, K]."""
    _tensor(q_dy_t, "q_dy_t", _FP8, (2,))
    _tensor(s_dy, "s_dy", _F32)
    _tensor(q_x_t, "q_x_t", _FP8, (2,))
    _tensor(s_x, "s_x", _F32)
    _tensor(out, "out", _BF16)
    N, Mp = q_dy_t.shape
    K = q_x_t.shape[0]
    if q_x_t.shape[1] != Mp:
        raise ValueError("q_dy_t and q_x_t differ in tokens (%d, %d)" % (Mp, q_x_t.shape[1]))
    _multiple(N, "N")
    _multiple(K, "K")
    if Mp % WGRAD_TOKEN_GROUP or Mp == 0:
        raise ValueError("Mp = %d is not a positive multiple of %d" % (Mp, WGRAD_TOKEN_GROUP))
    _numel(s_dy, (Mp // TILE) * N, "s_dy")
    _numel(s_x, (Mp // TILE) * K, "s_x")
    _numel(out, N * K, "out")
    dev = _device_of(q_dy_t=q_dy_t, s_dy=s_dy, q_x_t=q_x_t, s_x=s_x, out=out)
    if out is None:
        out = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    with torch.cuda.device(dev):
        _check(lib().fp8_gemm_wgrad(_p(q_dy_t), _p(s_dy), _p(q_x_t), _p(s_x), _p(out), N, K, Mp,
                                    _stream(stream, dev)), "fp8_gemm_wgrad")
    return out


MX_ATOM = 512  # bytes of E8M0 scales per 128-row tile and 128-deep slab


def fp8_mx_scales_act(sa: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Power-of-two 1x128 scales sa [M, K/128] f32 -> E8M0 atoms [ceil(M/128), K/128, 512] uint8."""
    _tensor(sa, "sa", _F32, (2,))
    M, nkb = sa.shape
    mt = (M + TILE - 1) // TILE
    _tensor(out, "out", (torch.uint8,))
    _numel(out, mt * nkb * MX_ATOM, "out")
    dev = _device_of(sa=sa, out=out)
    if out is None:
        out = torch.empty((mt, nkb, MX_ATOM), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        _check(lib().fp8_mx_scales_act(_p(sa), M, nkb * TILE, _p(out), _stream(stream, dev)), "fp8_mx_scales_act")
    return out


def fp8_mx_scales_w(sb: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Power-of-two 128x128 block scales sb [(G,) N/128, K/128] f32 -> E8M0 atoms [G*N/128, K/128, 512]."""
    _tensor(sb, "sb", _F32, (2, 3))
    G, nnb, nkb = (1,) + tuple(sb.shape) if sb.dim() == 2 else tuple(sb.shape)
    _tensor(out, "out", (torch.uint8,))
    _numel(out, G * nnb * nkb * MX_ATOM, "out")
    dev = _device_of(sb=sb, out=out)
    if out is None:
        out = torch.empty((G * nnb, nkb, MX_ATOM), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        _check(lib().fp8_mx_scales_w(_p(sb), G, nnb * TILE, nkb * TILE, _p(out), _stream(stream, dev)),
               "fp8_mx_scales_w")
    return out


def fp8_gemm_mx(qa, sfa_mx, qb, sfb_mx, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """C[M,N] (bf16) = A * B^T with power-of-two scales applied by the tensor cores: qa [M,K], qb [N,K]
    E4M3 from the _ue8m0 quantizers, their scales converted by fp8_mx_scales_act / fp8_mx_scales_w."""
    _tensor(qa, "qa", _FP8, (2,))
    _tensor(qb, "qb", _FP8, (2,))
    _tensor(sfa_mx, "sfa_mx", (torch.uint8,))
    _tensor(sfb_mx, "sfb_mx", (torch.uint8,))
    _tensor(out, "out", _BF16)
    M, K = qa.shape
    N = qb.shape[0]
    if qb.shape[1] != K:
        raise ValueError("qa and qb differ in K (%d, %d)" % (K, qb.shape[1]))
    _multiple(N, "N")
    _multiple(K, "K")
    _numel(sfa_mx, ((M + TILE - 1) // TILE) * (K // TILE) * MX_ATOM, "sfa_mx")
    _numel(sfb_mx, (N // TILE) * (K // TILE) * MX_ATOM, "sfb_mx")
    _numel(out, M * N, "out")
    dev = _device_of(qa=qa, sfa_mx=sfa_mx, qb=qb, sfb_mx=sfb_mx, out=out)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    with torch.cuda.device(dev):
        _check(lib().fp8_gemm_mx(_p(qa), _p(sfa_mx), _p(qb), _p(sfb_mx), _p(out), M, N, K, _stream(stream, dev)),
               "fp8_gemm_mx")
    return out


def fp8_grouped_gemm_mx_contiguous(qa, sfa_mx, qb, sfb_mx, m_indices, out: torch.Tensor | None = None, stream=None):
    """Contiguous-layout grouped GEMM with power-of-two scales applied by the tensor cores:
    qa [M_tot,K], qb [E,N,K] E4M3, their scale atoms, m_indices int32 [M_tot/128]."""
    _tensor(qa, "qa", _FP8, (2,))
    _tensor(qb, "qb", _FP8, (3,))
    _tensor(sfa_mx, "sfa_mx", (torch.uint8,))
    _tensor(sfb_mx, "sfb_mx", (torch.uint8,))
    _tensor(m_indices, "m_indices", _I32)
    _tensor(out, "out", _BF16)
    M_tot, K = qa.shape
    E, N, K2 = qb.shape
    if K2 != K:
        raise ValueError("qa and qb differ in K (%d, %d)" % (K, K2))
    _multiple(M_tot, "M_tot")
    _multiple(N, "N")
    _multiple(K, "K")
    _numel(sfa_mx, (M_tot // TILE) * (K // TILE) * MX_ATOM, "sfa_mx")
    _numel(sfb_mx, E * (N // TILE) * (K // TILE) * MX_ATOM, "sfb_mx")
    _numel(m_indices, M_tot // TILE, "m_indices")
    _numel(out, M_tot * N, "out")
    dev = _device_of(qa=qa, sfa_mx=sfa_mx, qb=qb, sfb_mx=sfb_mx, m_indices=m_indices, out=out)
    if out is None:
        out = torch.empty((M_tot, N), dtype=torch.bfloat16, device=dev)
    with torch.cuda.device(dev):
        _check(lib().fp8_grouped_gemm_mx_contiguous(_p(qa), _p(sfa_mx), _p(qb), _p(sfb_mx), _p(m_indices), _p(out),
                                                    M_tot, N, K, E, _stream(stream, dev)),
               "fp8_grouped_gemm_mx_contiguous")
    return out


def fp8_grouped_gemm_mx_masked(qa, sfa_mx, qb, sfb_mx, masked_m, out: torch.Tensor | None = None, stream=None):
    """Masked-layout grouped GEMM with power-of-two scales applied by the tensor cores:
    qa [E,cap,K], qb [E,N,K] E4M3, their scale atoms, masked_m int32 [E]; rows >= masked_m[e] unwritten."""
    _tensor(qa, "qa", _FP8, (3,))
    _tensor(qb, "qb", _FP8, (3,))
    _tensor(sfa_mx, "sfa_mx", (torch.uint8,))
    _tensor(sfb_mx, "sfb_mx", (torch.uint8,))
    _tensor(masked_m, "masked_m", _I32)
    _tensor(out, "out", _BF16)
    E, cap, K = qa.shape
    E2, N, K2 = qb.shape
    if E2 != E or K2 != K:
        raise ValueError("qa [E=%d, K=%d] and qb [E=%d, K=%d] do not agree" % (E, K, E2, K2))
    _multiple(cap, "cap")
    _multiple(N, "N")
    _multiple(K, "K")
    _numel(sfa_mx, E * (cap // TILE) * (K // TILE) * MX_ATOM, "sfa_mx")
    _numel(sfb_mx, E * (N // TILE) * (K // TILE) * MX_ATOM, "sfb_mx")
    _numel(masked_m, E, "masked_m")
    _numel(out, E * cap * N, "out")
    dev = _device_of(qa=qa, sfa_mx=sfa_mx, qb=qb, sfb_mx=sfb_mx, masked_m=masked_m, out=out)
    if out is None:
        out = torch.empty((E, cap, N), dtype=torch.bfloat16, device=dev)
    with torch.cuda.device(dev):
        _check(lib().fp8_grouped_gemm_mx_masked(_p(qa), _p(sfa_mx), _p(qb), _p(sfb_mx), _p(masked_m), _p(out), E,
                                                cap, N, K, _stream(stream, dev)), "fp8_grouped_gemm_mx_masked")
    return out


def fp8_grouped_gemm_contiguous(qa, sa, qb, sb, m_indices, out: torch.Tensor | None = None, stream=None):
    """Contiguous-layout grouped GEMM: C[M_tot,N]; block b uses expert m_indices[b].

    qa [M_tot,K], sa [M_tot,K/128], qb [E,N,K], sb [E,N/128,K/128], m_indices int32 [M_tot/128]."""
    _tensor(qa, "qa", _FP8, (2,))
    _tensor(sa, "sa", _F32)
    _tensor(qb, "qb", _FP8, (3,))
    _tensor(sb, "sb", _F32)
    _tensor(m_indices, "m_indices", _I32)
    _tensor(out, "out", _BF16)
    M_tot, K = qa.shape
    E, N, K2 = qb.shape
    if K2 != K:
        raise ValueError("qa and qb differ in K (%d, %d)" % (K, K2))
    _multiple(M_tot, "M_tot")
    _multiple(N, "N")
    _multiple(K, "K")
    _numel(sa, M_tot * (K // TILE), "sa")
    _numel(sb, E * (N // TILE) * (K // TILE), "sb")
    _numel(m_indices, M_tot // TILE, "m_indices")
    _numel(out, M_tot * N, "out")
    dev = _device_of(qa=qa, sa=sa, qb=qb, sb=sb, m_indices=m_indices, out=out)
    if out is None:
        out = torch.empty((M_tot, N), dtype=torch.bfloat16, device=dev)
    with torch.cuda.device(dev):
        _check(lib().fp8_grouped_gemm_contiguous(_p(qa), _p(sa), _p(qb), _p(sb), _p(m_indices), _p(out), M_tot, N, K,
                                                 E, _stream(stream, dev)), "fp8_grouped_gemm_contiguous")
    return out


def fp8_grouped_gemm_masked(qa, sa, qb, sb, masked_m, expected_m: int = 0, out: torch.Tensor | None = None,
                            stream=None):
    """Masked-layout grouped GEMM: C[E,cap,N]; rows >= masked_m[e] are left unwritten.

    qa [E,cap,K], sa [E,cap,K/128], qb [E,N,K], sb [E,N/128,K/128], masked_m int32 [E]."""
    _tensor(qa, "qa", _FP8, (3,))
    _tensor(sa, "sa", _F32)
    _tensor(qb, "qb", _FP8, (3,))
    _tensor(sb, "sb", _F32)
    _tensor(masked_m, "masked_m", _I32)
    _tensor(out, "out", _BF16)
    E, cap, K = qa.shape
    E2, N, K2 = qb.shape
    if E2 != E or K2 != K:
        raise ValueError("qa [E=%d, K=%d] and qb [E=%d, K=%d] do not agree" % (E, K, E2, K2))
    _multiple(cap, "cap")
    _multiple(N, "N")
    _multiple(K, "K")
    _numel(sa, E * cap * (K // TILE), "sa")
    _numel(sb, E * (N // TILE) * (K // TILE), "sb")
    _numel(masked_m, E, "masked_m")
    _numel(out, E * cap * N, "out")
    dev = _device_of(qa=qa, sa=sa, qb=qb, sb=sb, masked_m=masked_m, out=out)
    if out is None:
        out = torch.empty((E, cap, N), dtype=torch.bfloat16, device=dev)
    with torch.cuda.device(dev):
        _check(lib().fp8_grouped_gemm_masked(_p(qa), _p(sa), _p(qb), _p(sb), _p(masked_m), _p(out), E, cap, N, K,
                                             int(expected_m), _stream(stream, dev)), "fp8_grouped_gemm_masked")
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
