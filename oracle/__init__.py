"""numpy front end of the plain C oracle (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package.  The CUDA library never reaches it, and it imports nothing
from the CUDA package.  All arrays are numpy; bf16 tensors travel as their uint16 bit
patterns.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None

_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64

ROW, COL = 1, 2
ROW_MAJOR, COL_MAJOR = 0, 1


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(os.path.abspath(path))
        L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_double.restype = ctypes.c_double
        L.oracle_double_to_bf16.argtypes = [ctypes.c_double]
        L.oracle_double_to_bf16.restype = ctypes.c_uint16
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_e4m3_encode.argtypes = [ctypes.c_double]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e8m0_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e8m0_decode.restype = ctypes.c_double
        L.oracle_floor_log2.argtypes = [ctypes.c_double]
        L.oracle_floor_log2.restype = ctypes.c_int
        L.oracle_mx_scale_byte.argtypes = [ctypes.c_double]
        L.oracle_mx_scale_byte.restype = ctypes.c_uint8
        L.oracle_e4m3_encode_f64_array.argtypes = [_f64p, _i64, _u8p]
        L.oracle_e4m3_encode_f32_array.argtypes = [_f32p, _i64, _u8p]
        L.oracle_double_to_bf16_array.argtypes = [_f64p, _i64, _u16p]
        L.oracle_mx_quantize.argtypes = [_u16p, _i64, _i64, _i64, ctypes.c_int,
                                         _u8p, _u8p, _u8p, _u8p]
        L.oracle_mx_dequantize.argtypes = [_u8p, _u8p, _i64, _i64, _i64, ctypes.c_int, _u16p]
        L.oracle_per_group_quant.argtypes = [_u16p, _i64, _i64, _i32p, ctypes.c_int32,
                                             ctypes.c_int, _u8p, _f32p]
        L.oracle_group_bounds.argtypes = [_i32p, ctypes.c_int32, _i64, _i64p, _i64p]
        L.oracle_transpose_u8.argtypes = [_u8p, _i64, _i64, _i64, _u8p]
        L.oracle_mx_scales_blocked_bytes.argtypes = [_i64, _i64, _i64, ctypes.c_int32]
        L.oracle_mx_scales_blocked_bytes.restype = ctypes.c_int64
        L.oracle_mx_scales_to_blocked.argtypes = [_u8p, _i64, _i64, _i64, _i32p, ctypes.c_int32, _u8p]
        L.oracle_mx_grouped_gemm.argtypes = [_u8p, _u8p, _u8p, _u8p, _i32p, ctypes.c_int32, _i64, _i64,
                                             _i64, _f64p, _f64p]
        L.oracle_mx_grouped_gemm.restype = None
        for name in ("oracle_e4m3_encode_f64_array", "oracle_e4m3_encode_f32_array",
                     "oracle_double_to_bf16_array", "oracle_mx_quantize",
                     "oracle_mx_dequantize", "oracle_per_group_quant", "oracle_group_bounds",
                     "oracle_transpose_u8", "oracle_mx_scales_to_blocked"):
            getattr(L, name).restype = None
        _LIB = L
    return _LIB


def _ptr(a: np.ndarray, typ):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(typ)


# ---- scalar formats ----------------------------------------------------------------

def bf16_to_double(bits) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    with np.errstate(invalid="ignore"):
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def double_to_bf16(v) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    lib().oracle_double_to_bf16_array(_ptr(v, _f64p), v.size, _ptr(out, _u16p))
    return out


def e4m3_decode(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    table = np.array([lib().oracle_e4m3_decode(c) for c in range(256)], dtype=np.float64)
    return table[codes]


def e4m3_encode(v) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().oracle_e4m3_encode_f64_array(_ptr(v, _f64p), v.size, _ptr(out, _u8p))
    return out


def e4m3_encode_f32(v) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().oracle_e4m3_encode_f32_array(_ptr(v, _f32p), v.size, _ptr(out, _u8p))
    return out


def e8m0_decode(b: int) -> float:
    return lib().oracle_e8m0_decode(int(b))


def mx_scale_byte(amax: float) -> int:
    return int(lib().oracle_mx_scale_byte(float(amax)))


def floor_log2(a: float) -> int:
    return int(lib().oracle_floor_log2(float(a)))


# ---- MX quantize / dequantize -------------------------------------------------------

def mx_quantize(x_bits: np.ndarray, axes: int = ROW):
    """x_bits: (rows, cols) or (batch, rows, cols) uint16.  Returns a dict with the
    outputs the requested axes produce (q_row, s_row, q_col, s_col), batch-shaped
    like the input."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    squeeze = x.ndim == 2
    if squeeze:
        x = x[None]
    batch, rows, cols = x.shape
    assert cols % 32 == 0 and (rows % 32 == 0 or not axes & COL)
    out = {}
    q_row = np.empty((batch, rows, cols), np.uint8) if axes & ROW else np.empty(1, np.uint8)
    s_row = np.empty((batch, rows, cols // 32), np.uint8) if axes & ROW else np.empty(1, np.uint8)
    q_col = np.empty((batch, cols, rows), np.uint8) if axes & COL else np.empty(1, np.uint8)
    s_col = np.empty((batch, cols, rows // 32), np.uint8) if axes & COL else np.empty(1, np.uint8)
    lib().oracle_mx_quantize(_ptr(x, _u16p), batch, rows, cols, axes, _ptr(q_row, _u8p),
                             _ptr(s_row, _u8p), _ptr(q_col, _u8p), _ptr(s_col, _u8p))
    if axes & ROW:
        out["q_row"], out["s_row"] = (q_row[0], s_row[0]) if squeeze else (q_row, s_row)
    if axes & COL:
        out["q_col"], out["s_col"] = (q_col[0], s_col[0]) if squeeze else (q_col, s_col)
    return out


def mx_dequantize(q: np.ndarray, s: np.ndarray, batch: int, rows: int, cols: int,
                  axis: int = ROW) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    s = np.ascontiguousarray(s, dtype=np.uint8)
    y = np.empty((batch, rows, cols), np.uint16)
    lib().oracle_mx_dequantize(_ptr(q, _u8p), _ptr(s, _u8p), batch, rows, cols, axis,
                               _ptr(y, _u16p))
    return y if batch > 1 else y[0]


# ---- per-group rowwise -----------------------------------------------------------------

def group_bounds(offs, M: int):
    offs = np.ascontiguousarray(offs, dtype=np.int32)
    G = offs.size
    start = np.empty(G, np.int64)
    end = np.empty(G, np.int64)
    lib().oracle_group_bounds(_ptr(offs, _i32p), G, M, _ptr(start, _i64p), _ptr(end, _i64p))
    return start, end


def per_group_quant(x_bits: np.ndarray, offs, layout: int = ROW_MAJOR, q_init=None):
    """x_bits: (M, K) uint16.  Returns (q, scales); q is (M, K) for the row-major
    layout and (K, M) for the column-major one.  Bytes of rows outside every group
    keep the value of ``q_init`` (default 0)."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    M, K = x.shape
    offs = np.ascontiguousarray(offs, dtype=np.int32)
    G = offs.size
    shape = (M, K) if layout == ROW_MAJOR else (K, M)
    if q_init is None:
        q = np.zeros(shape, np.uint8)
    else:
        q = np.ascontiguousarray(np.array(q_init, dtype=np.uint8).reshape(shape))
    scales = np.empty((G, K), np.float32)
    lib().oracle_per_group_quant(_ptr(x, _u16p), M, K, _ptr(offs, _i32p), G, layout,
                                 _ptr(q, _u8p), _ptr(scales, _f32p))
    return q, scales


# ---- layouts the scaled grouped GEMM consumes -----------------------------------------

def transpose_u8(src: np.ndarray) -> np.ndarray:
    """(rows, cols) or (batch, rows, cols) uint8 -> its per-matrix transpose."""
    x = np.ascontiguousarray(src, dtype=np.uint8)
    squeeze = x.ndim == 2
    if squeeze:
        x = x[None]
    b, r, c = x.shape
    out = np.empty((b, c, r), np.uint8)
    lib().oracle_transpose_u8(_ptr(x, _u8p), b, r, c, _ptr(out, _u8p))
    return out[0] if squeeze else out


def mx_scales_blocked_bytes(batch: int, rows: int, n_k: int, G: int = 0) -> int:
    return int(lib().oracle_mx_scales_blocked_bytes(batch, rows, n_k, G))


def mx_scales_to_blocked(s: np.ndarray, offs=None, fill: int = 0) -> np.ndarray:
    """E8M0 scales (rows, n_k) or (batch, rows, n_k) -> the blocked 128 x 4 tile layout
    (a flat uint8 array of mx_scales_blocked_bytes); with offs (batch 1), every
    group's rows padded to a multiple of 128 on their own.  Bytes past the used
    tiles keep `fill`."""
    x = np.ascontiguousarray(s, dtype=np.uint8)
    if x.ndim == 2:
        x = x[None]
    b, r, k = x.shape
    if offs is None:
        G, o = 0, np.zeros(1, np.int32)
    else:
        o = np.ascontiguousarray(offs, dtype=np.int32)
        G = o.size
        assert b == 1
    out = np.full(mx_scales_blocked_bytes(b, r, k, G), fill, np.uint8)
    lib().oracle_mx_scales_to_blocked(_ptr(x, _u8p), b, r, k, _ptr(o, _i32p), G, _ptr(out, _u8p))
    return out


# ---- MXFP8 grouped GEMM ----------------------------------------------------------------------

def mx_grouped_gemm(qa, sa, qb, sb, offs, fill: float = np.nan):
    """qa (M, K), sa (M, K/32): MX row layout of the tokens; qb (G, N, K), sb (G, N, K/32):
    the experts.  Returns (out, abs_sum), (M, N) doubles: the exact per-group product of
    the dequantized operands and sum |a_k b_k|; rows in no group keep `fill`."""
    qa = np.ascontiguousarray(qa, np.uint8)
    sa = np.ascontiguousarray(sa, np.uint8)
    qb = np.ascontiguousarray(qb, np.uint8)
    sb = np.ascontiguousarray(sb, np.uint8)
    offs = np.ascontiguousarray(offs, np.int32)
    M, K = qa.shape
    G, N, K2 = qb.shape
    assert K2 == K and K % 32 == 0 and G == offs.size
    out = np.full((M, N), fill, np.float64)
    mag = np.full((M, N), fill, np.float64)
    lib().oracle_mx_grouped_gemm(_ptr(qa, _u8p), _ptr(sa, _u8p), _ptr(qb, _u8p), _ptr(sb, _u8p),
                                 _ptr(offs, _i32p), G, M, N, K, _ptr(out, _f64p), _ptr(mag, _f64p))
    return out, mag


def per_group_quant_batched(x_bits: np.ndarray, layout: int = ROW_MAJOR):
    """x_bits (E, M, K) uint16, every matrix its own group (the 3-D left operand of a
    grouped GEMM).  Returns (q, scales): q (E, M, K) for the row-major layout, (E, K, M)
    (each matrix column-major) for the column-major one; scales (E, K).  Each matrix is
    oracle_per_group_quant with the single group [0, M)."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    E, M, K = x.shape
    qs, ss = [], []
    for e in range(E):
        q, s = per_group_quant(x[e], np.array([M], np.int32), layout)
        qs.append(q)
        ss.append(s[0])
    shape = (E, M, K) if layout == ROW_MAJOR else (E, K, M)
    return (np.stack(qs) if E else np.zeros(shape, np.uint8)), (np.stack(ss) if E else np.zeros((0, K), np.float32))
