"""CPU oracle for fine-grained FP8 quantization and the block-scaled FP8 GEMM.

TEST INFRASTRUCTURE ONLY.  The product library never imports, links or runs
anything in this package; only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may.  It shares no code with the CUDA path:
the arithmetic lives in ``fp8q_oracle.c`` (plain C, IEEE float, no fast-math),
and this module only marshals numpy arrays into it.

What each function computes, and the passage it follows, is documented beside
the C function it wraps.  Parity pins for every function live in
``tests/test_oracle_*.py``; none of them is left unpinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SOURCES = [_HERE / "fp8q_oracle.c", _HERE / "e4m3_search_check.c"]
_LIB_PATH = _HERE / "liboracle.so"
_lib = None

TILE = 128


def build(force: bool = False) -> Path:
    """Compile the oracle into ``liboracle.so`` (gcc, OpenMP, IEEE float)."""
    newest = max(p.stat().st_mtime for p in _SOURCES)
    if not force and _LIB_PATH.exists() and _LIB_PATH.stat().st_mtime >= newest:
        return _LIB_PATH
    tmp = _LIB_PATH.with_suffix(".so.tmp%d" % os.getpid())
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
           "-Wall", "-Wextra", "-o", str(tmp)] + [str(p) for p in _SOURCES] + ["-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(str(_LIB_PATH))
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    lib.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.orc_e4m3_decode.restype = ctypes.c_double
    lib.orc_e4m3_encode.argtypes = [ctypes.c_float]
    lib.orc_e4m3_encode.restype = ctypes.c_uint8
    lib.orc_e4m3_encode_by_search.argtypes = [ctypes.c_float]
    lib.orc_e4m3_encode_by_search.restype = ctypes.c_uint8
    lib.orc_e4m3_encode_array.argtypes = [P, I64, P]
    lib.orc_e4m3_encode_array.restype = None
    lib.orc_e4m3_decode_table.argtypes = [P]
    lib.orc_e4m3_decode_table.restype = None
    lib.orc_e4m3_exhaustive_check.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64,
                                              ctypes.POINTER(ctypes.c_uint32)]
    lib.orc_e4m3_exhaustive_check.restype = I64
    lib.orc_quant_act_1x128.argtypes = [P, I64, I64, P, P]
    lib.orc_quant_w_128x128.argtypes = [P, I64, I64, I64, P, P]
    lib.orc_quant_tensor.argtypes = [P, I64, P, P]
    lib.orc_quant_with_scale.argtypes = [P, I64, ctypes.c_float, P]
    lib.orc_quant_with_scale.restype = ctypes.c_int
    lib.orc_quant_act_1x128_ue8m0.argtypes = [P, I64, I64, P, P]
    lib.orc_quant_act_1x128_ue8m0.restype = ctypes.c_int
    lib.orc_quant_w_128x128_ue8m0.argtypes = [P, I64, I64, I64, P, P]
    lib.orc_quant_w_128x128_ue8m0.restype = ctypes.c_int
    lib.orc_round_bf16.argtypes = [P, I64, P]
    lib.orc_round_bf16.restype = None
    lib.orc_swiglu_bf16.argtypes = [P, I64, I64, P]
    lib.orc_swiglu_bf16.restype = ctypes.c_int
    lib.orc_quant_act_128x1.argtypes = [P, I64, I64, P, P]
    lib.orc_quant_act_128x1.restype = ctypes.c_int
    lib.orc_gemm_1d1d.argtypes = [P, P, P, P, I64, I64, I64, P, I64, P]
    lib.orc_gemm_1d1d.restype = ctypes.c_int
    lib.orc_gemm_blockscaled.argtypes = [P, P, P, P, I64, I64, I64, P, I64, P]
    lib.orc_grouped_contiguous.argtypes = [P, P, P, P, P, I64, I64, I64, I64, P, I64, P]
    lib.orc_grouped_masked.argtypes = [P, P, P, P, P, I64, I64, I64, I64, P, I64, P]
    lib.orc_gemm_limited_acc.argtypes = [P, P, P, P, I64, I64, I64, ctypes.c_int, I64, I64, P, I64, P]
    for name in ("orc_quant_act_1x128", "orc_quant_w_128x128", "orc_quant_tensor", "orc_gemm_blockscaled",
                 "orc_grouped_contiguous", "orc_grouped_masked", "orc_gemm_limited_acc"):
        getattr(lib, name).restype = ctypes.c_int
    lib.orc_num_threads.restype = ctypes.c_int
    _lib = lib
    return lib


_DTYPES = {"u8": np.uint8, "f32": np.float32, "f64": np.float64, "i32": np.int32, "i64": np.int64,
           "u16": np.uint16}


def _ptr(a: np.ndarray | None, kind: str | None = None):
    if a is None:
        return None
    if kind is not None and a.dtype != _DTYPES[kind]:
        raise TypeError("oracle expects %s, got %s" % (kind, a.dtype))
    if not a.flags["C_CONTIGUOUS"]:
        raise ValueError("oracle inputs must be C-contiguous")
    return ctypes.c_void_p(a.ctypes.data)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError("%s: oracle rejected the arguments (code %d)" % (what, rc))


def _bf16(a: np.ndarray) -> np.ndarray:
    assert a.dtype == np.uint16, "bf16 inputs are passed as their uint16 bit patterns"
    return np.ascontiguousarray(a)


def num_threads() -> int:
    return int(_load().orc_num_threads())


# --------------------------------------------------------------------------- E4M3
def e4m3_decode(code: int) -> float:
    """Value of one E4M3FN code (1-4-3 layout, bias 7, NaN = S.1111.111)."""
    return float(_load().orc_e4m3_decode(int(code) & 0xFF))


def e4m3_decode_table() -> np.ndarray:
    out = np.empty(256, dtype=np.float64)
    _load().orc_e4m3_decode_table(_ptr(out))
    return out


def e4m3_encode(v: float) -> int:
    """RNE onto the E4M3 grid, saturating at +-448 (bit-manipulation encoder)."""
    return int(_load().orc_e4m3_encode(ctypes.c_float(v)))


def e4m3_encode_array(v: np.ndarray) -> np.ndarray:
    """Vector form of :func:`e4m3_encode` over a float32 array."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    _load().orc_e4m3_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def e4m3_encode_by_search(v: float) -> int:
    """Independent nearest-value-search encoder (test cross-check only)."""
    return int(_load().orc_e4m3_encode_by_search(ctypes.c_float(v)))


def e4m3_exhaustive_check(first: int = 0, end: int = 1 << 32, stride: int = 1):
    bad = ctypes.c_uint32(0)
    n = _load().orc_e4m3_exhaustive_check(first, end, stride, ctypes.byref(bad))
    return int(n), int(bad.value)


# --------------------------------------------------------------------------- quantizers
def quant_act_1x128(x_bf16: np.ndarray):
    """[M,K] bf16 bits -> (q [M,K] uint8 E4M3 codes, s [M,K/128] float32)."""
    x = _bf16(x_bf16)
    M, K = x.shape
    q = np.empty((M, K), dtype=np.uint8)
    s = np.empty((M, K // TILE), dtype=np.float32)
    _check(_load().orc_quant_act_1x128(_ptr(x), M, K, _ptr(q), _ptr(s)), "quant_act_1x128")
    return q, s


def quant_act_1x128_ue8m0(x_bf16: np.ndarray):
    """1x128 tiles with power-of-two (UE8M0) scales -> (q [M,K], s [M,K/128] f32, each 2^e)."""
    x = _bf16(x_bf16)
    M, K = x.shape
    q = np.empty((M, K), dtype=np.uint8)
    s = np.empty((M, K // TILE), dtype=np.float32)
    _check(_load().orc_quant_act_1x128_ue8m0(_ptr(x), M, K, _ptr(q), _ptr(s)), "quant_act_1x128_ue8m0")
    return q, s


def quant_w_128x128_ue8m0(w_bf16: np.ndarray):
    """128x128 blocks with power-of-two (UE8M0) scales, [N,K] or [G,N,K]."""
    w = _bf16(w_bf16)
    squeeze = w.ndim == 2
    if squeeze:
        w = w[None]
    G, N, K = w.shape
    q = np.empty((G, N, K), dtype=np.uint8)
    s = np.empty((G, N // TILE, K // TILE), dtype=np.float32)
    _check(_load().orc_quant_w_128x128_ue8m0(_ptr(w), G, N, K, _ptr(q), _ptr(s)), "quant_w_128x128_ue8m0")
    return (q[0], s[0]) if squeeze else (q, s)


def quant_act_128x1(x_bf16: np.ndarray):
    """[M,K] bf16 bits -> (q [M,K] codes, s [ceil(M/128),K] float32): groups of
    128 tokens per channel (the token-axis tiles of the weight gradient)."""
    x = _bf16(x_bf16)
    M, K = x.shape
    q = np.empty((M, K), dtype=np.uint8)
    s = np.empty(((M + TILE - 1) // TILE, K), dtype=np.float32)
    _check(_load().orc_quant_act_128x1(_ptr(x), M, K, _ptr(q), _ptr(s)), "quant_act_128x1")
    return q, s


def quant_w_128x128(w_bf16: np.ndarray):
    """[N,K] or [G,N,K] bf16 bits -> (q, s [.., N/128, K/128])."""
    w = _bf16(w_bf16)
    squeeze = w.ndim == 2
    if squeeze:
        w = w[None]
    G, N, K = w.shape
    q = np.empty((G, N, K), dtype=np.uint8)
    s = np.empty((G, N // TILE, K // TILE), dtype=np.float32)
    _check(_load().orc_quant_w_128x128(_ptr(w), G, N, K, _ptr(q), _ptr(s)), "quant_w_128x128")
    return (q[0], s[0]) if squeeze else (q, s)


def quant_tensor(x_bf16: np.ndarray):
    """Per-tensor E4M3 quantization (one scale) -> (q, s: float)."""
    x = _bf16(x_bf16)
    q = np.empty(x.shape, dtype=np.uint8)
    s = np.empty(1, dtype=np.float32)
    _check(_load().orc_quant_tensor(_ptr(x), x.size, _ptr(q), _ptr(s)), "quant_tensor")
    return q, float(s[0])


def quant_with_scale(x_bf16: np.ndarray, s: float) -> np.ndarray:
    """E4M3 codes of fl32(x / s) for a given scale s (delayed scaling)."""
    x = _bf16(x_bf16)
    q = np.empty(x.shape, dtype=np.uint8)
    _check(_load().orc_quant_with_scale(_ptr(x), x.size, float(s), _ptr(q)), "quant_with_scale")
    return q


# --------------------------------------------------------------------------- GEMMs
def _shapes(*pairs):
    for a, shape in zip(pairs[0::2], pairs[1::2]):
        if tuple(np.shape(a)) != tuple(shape):
            raise ValueError("oracle: expected shape %s, got %s" % (shape, np.shape(a)))


def _rows(rows):
    if rows is None:
        return None, 0
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    return r, r.size


def gemm_blockscaled(qa, sa, qb, sb, rows=None) -> np.ndarray:
    """float64 C = A * B^T with per-128-slab scaling; optional row subset."""
    M, K = qa.shape
    N = qb.shape[0]
    _shapes(sa, (M, K // TILE), qb, (N, K), sb, (N // TILE, K // TILE))
    r, nr = _rows(rows)
    C = np.empty((nr if r is not None else M, N), dtype=np.float64)
    _check(_load().orc_gemm_blockscaled(_ptr(qa, "u8"), _ptr(sa, "f32"), _ptr(qb, "u8"), _ptr(sb, "f32"), M, N, K, _ptr(r), nr, _ptr(C)),
           "gemm_blockscaled")
    return C


def gemm_1d1d(qa, sa, qb, sb, rows=None) -> np.ndarray:
    """float64 C = A * B^T with per-row, per-slab scales on both operands
    (sa [M,K/128], sb [N,K/128]); optional row subset."""
    M, K = qa.shape
    N = qb.shape[0]
    _shapes(sa, (M, K // TILE), qb, (N, K), sb, (N, K // TILE))
    r, nr = _rows(rows)
    C = np.empty((nr if r is not None else M, N), dtype=np.float64)
    _check(_load().orc_gemm_1d1d(_ptr(np.ascontiguousarray(qa), "u8"), _ptr(np.ascontiguousarray(sa), "f32"),
                                 _ptr(np.ascontiguousarray(qb), "u8"), _ptr(np.ascontiguousarray(sb), "f32"),
                                 M, N, K, _ptr(r), nr, _ptr(C)), "gemm_1d1d")
    return C


def wgrad(q_dy, s_dy, q_x, s_x, rows=None) -> np.ndarray:
    """dW [N,K] = dY^T X from token-axis quantized dY [M,N] and X [M,K]
    (quant_act_128x1 of each; M a multiple of 128).  Rows index N."""
    return gemm_1d1d(np.ascontiguousarray(q_dy.T), np.ascontiguousarray(s_dy.T),
                     np.ascontiguousarray(q_x.T), np.ascontiguousarray(s_x.T), rows)


def dgrad(q_dy, s_dy, q_w, s_w, rows=None) -> np.ndarray:
    """dX [M,K] = dY W from 1x128-quantized dY [M,N] and 128x128-quantized
    W [N,K]: the forward GEMM with W's codes and block scales transposed."""
    return gemm_blockscaled(q_dy, s_dy, np.ascontiguousarray(q_w.T), np.ascontiguousarray(s_w.T), rows)


def round_bf16(v: np.ndarray) -> np.ndarray:
    """float64 values -> bf16 bit patterns, one round-to-nearest-even step."""
    x = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().orc_round_bf16(_ptr(x), x.size, _ptr(out))
    return out


def masked_moe_chain(a_bits, b1_bits, b2_bits, masked_m) -> np.ndarray:
    """The masked MoE decode as one chain: 1x128 quantization of A [E,cap,K1], masked
    GEMM1 with 128x128-quantized B1 [E,2I,K1], bf16 rounding of its output,
    SwiGLU, 1x128 requantization, masked GEMM2 with B2 [E,N2,I].  Returns the
    float64 GEMM2 output [E,cap,N2]; rows at or past masked_m[e] are NaN."""
    E, cap, K1 = a_bits.shape
    qa, sa = quant_act_1x128(a_bits.reshape(E * cap, K1))
    qb1, sb1 = quant_w_128x128(b1_bits)
    c1 = grouped_masked(qa.reshape(E, cap, K1), sa.reshape(E, cap, K1 // TILE), qb1, sb1, masked_m)
    c1 = np.where(np.isnan(c1), 0.0, c1)  # rows past the count never reach GEMM2's valid rows
    h = swiglu_bf16(round_bf16(c1))
    inter = h.shape[-1]
    qh, sh = quant_act_1x128(h.reshape(E * cap, inter))
    qb2, sb2 = quant_w_128x128(b2_bits)
    return grouped_masked(qh.reshape(E, cap, inter), sh.reshape(E, cap, inter // TILE), qb2, sb2, masked_m)


def swiglu_bf16(c1_bf16: np.ndarray) -> np.ndarray:
    """[.., 2I] bf16 bits ([gate | up]) -> [.., I] bf16 bits of silu(gate) * up (double, one rounding)."""
    c1 = _bf16(c1_bf16)
    inter = c1.shape[-1] // 2
    if c1.shape[-1] != 2 * inter:
        raise ValueError("oracle: the last dimension must be even ([gate | up])")
    rows = c1.size // (2 * inter) if inter else 0
    h = np.empty(c1.shape[:-1] + (inter,), dtype=np.uint16)
    _check(_load().orc_swiglu_bf16(_ptr(c1), rows, inter, _ptr(h)), "swiglu_bf16")
    return h


def grouped_contiguous(qa, sa, qb, sb, m_indices, rows=None, out=None) -> np.ndarray:
    """Contiguous-layout grouped GEMM.  Rows of blocks with an out-of-range
    expert index keep the contents of ``out`` (NaN when ``out`` is None)."""
    M_tot, K = qa.shape
    E, N, _ = qb.shape
    _shapes(sa, (M_tot, K // TILE), qb, (E, N, K), sb, (E, N // TILE, K // TILE), m_indices, (M_tot // TILE,))
    r, nr = _rows(rows)
    mi = np.ascontiguousarray(m_indices, dtype=np.int32)
    shape = (nr if r is not None else M_tot, N)
    C = np.full(shape, np.nan) if out is None else out
    _check(_load().orc_grouped_contiguous(_ptr(qa, "u8"), _ptr(sa, "f32"), _ptr(qb, "u8"), _ptr(sb, "f32"), _ptr(mi), M_tot, N, K, E,
                                          _ptr(r), nr, _ptr(C)), "grouped_contiguous")
    return C


def grouped_masked(qa, sa, qb, sb, masked_m, rows=None, out=None) -> np.ndarray:
    """Masked-layout grouped GEMM on qa [E,cap,K].  Result [E,cap,N] (or
    [nrows,N] for a row subset, rows = flat e*cap+m); rows at or past
    masked_m[e] keep the contents of ``out`` (NaN when ``out`` is None)."""
    E, cap, K = qa.shape
    N = qb.shape[1]
    _shapes(sa, (E, cap, K // TILE), qb, (E, N, K), sb, (E, N // TILE, K // TILE), masked_m, (E,))
    r, nr = _rows(rows)
    mm = np.ascontiguousarray(masked_m, dtype=np.int32)
    shape = (nr, N) if r is not None else (E, cap, N)
    C = np.full(shape, np.nan) if out is None else out
    _check(_load().orc_grouped_masked(_ptr(qa, "u8"), _ptr(sa, "f32"), _ptr(qb, "u8"), _ptr(sb, "f32"), _ptr(mm), E, cap, N, K, _ptr(r), nr,
                                      _ptr(C)), "grouped_masked")
    return C


def gemm_limited_acc(qa, sa, qb, sb, p_bits=14, group=32, interval=0, rows=None) -> np.ndarray:
    """Limited-precision accumulation model (drift demonstration)."""
    M, K = qa.shape
    N = qb.shape[0]
    _shapes(sa, (M, K // TILE), qb, (N, K), sb, (N // TILE, K // TILE))
    r, nr = _rows(rows)
    C = np.empty((nr if r is not None else M, N), dtype=np.float64)
    _check(_load().orc_gemm_limited_acc(_ptr(qa, "u8"), _ptr(sa, "f32"), _ptr(qb, "u8"), _ptr(sb, "f32"), M, N, K, p_bits, group, interval,
                                        _ptr(r), nr, _ptr(C)), "gemm_limited_acc")
    return C
