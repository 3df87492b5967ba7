"""B200-native MXFP8 / per-group FP8 quantization for MoE expert-parallel training.

Thin Python binding over the C ABI of ``libmxq.so`` (declared in ``include/mxq.h``).
Functions carry the C names and only marshal arguments: they check that the torch
tensors they are given are CUDA tensors of the right dtype, shape and contiguity,
pass their device pointers and the current CUDA stream to the C entry point, and raise
``MxqError`` on a non-zero status.  Every step of the computation runs in the CUDA
kernels; there is no CPU or PyTorch fallback, and the first call raises if the
library has not been built.

Operations (see include/mxq.h for the exact arithmetic and layouts):
  mx_quantize / mx_dequantize -- the local quantize and dequantize around the MXFP8
    expert-parallel all-to-all (torchtitan "[mxfp8 MoE training] Support mxfp8 all to
    all in expert parallel", Summary).
  fp8_per_group_rowwise_quant -- per-group rowwise FP8 scaling (torchao "[moe
    training] fix uncoalesced global accesses in per group rowwise scaling kernel").
"""
from __future__ import annotations

import ctypes
import os

import torch

ROW, COL = 1, 2
ROW_MAJOR, COL_MAJOR = 0, 1

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmxq.so")
_LIB = None


class MxqError(RuntimeError):
    pass


def lib() -> ctypes.CDLL:
    """Load libmxq.so (built in-tree by ``build.py``).  Raises if it is missing."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise MxqError(f"{LIB_PATH} is missing: build it with "
                           "`python -m mxfp8_quantization_moe_mx_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, ci = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int
        L.mx_quantize.argtypes = [vp, i64, i64, i64, ci, vp, vp, vp, vp, vp]
        L.mx_dequantize.argtypes = [vp, vp, i64, i64, i64, ci, vp, vp]
        L.fp8_per_group_rowwise_quant.argtypes = [vp, i64, i64, vp, i32, ci, vp, vp, vp]
        L.mx_e4m3_encode_f32.argtypes = [vp, i64, vp, vp]
        L.mxq_transpose_u8.argtypes = [vp, i64, i64, i64, vp, vp]
        L.mxq_transpose_u8.restype = ci
        L.mx_scales_to_blocked.argtypes = [vp, i64, i64, i64, vp, i32, vp, vp]
        L.mx_scales_to_blocked.restype = ci
        L.mx_scales_blocked_bytes.argtypes = [i64, i64, i64, i32]
        L.mx_scales_blocked_bytes.restype = i64
        L.fp8_per_group_rowwise_quant_batched.argtypes = [vp, i64, i64, i64, ci, vp, vp, vp]
        L.fp8_per_group_rowwise_quant_batched.restype = ci
        L.mx_grouped_gemm.argtypes = [vp, vp, vp, vp, vp, i32, i64, i64, i64, vp, vp]
        L.mx_grouped_gemm.restype = ci
        for f in (L.mx_quantize, L.mx_dequantize, L.fp8_per_group_rowwise_quant,
                  L.mx_e4m3_encode_f32):
            f.restype = ci
        L.mxq_status_string.argtypes = [ci]
        L.mxq_status_string.restype = ctypes.c_char_p
        L.mxq_last_cuda_error.argtypes = []
        L.mxq_last_cuda_error.restype = ctypes.c_char_p
        L.mxq_wait_timeouts.argtypes = [ctypes.POINTER(ctypes.c_uint)]
        L.mxq_wait_timeouts.restype = ci
        L.mxq_wait_abandoned.argtypes = [ctypes.POINTER(ctypes.c_uint)]
        L.mxq_wait_abandoned.restype = ci
        L.mxq_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        L.mxq_set_wait_limit_ns.restype = ci
        ip = ctypes.POINTER(ci)
        L.fp8_per_group_rowwise_plan.argtypes = [i64, i64, i32, ci, ci, ip, ip, ip, ip, ip]
        L.fp8_per_group_rowwise_plan.restype = ci
        _LIB = L
    return _LIB


def _check(status: int) -> None:
    if status != 0:
        L = lib()
        msg = L.mxq_status_string(status).decode()
        if status == 5:
            msg += ": " + L.mxq_last_cuda_error().decode()
        raise MxqError(msg)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev(t: torch.Tensor, dtype, name: str, numel: int | None = None) -> int:
    if not isinstance(t, torch.Tensor):
        raise MxqError(f"{name} must be a torch tensor")
    if not t.is_cuda:
        raise MxqError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise MxqError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise MxqError(f"{name} must be contiguous")
    if numel is not None and t.numel() != numel:
        raise MxqError(f"{name} has {t.numel()} elements, expected {numel}")
    return t.data_ptr()


def _bsc(x: torch.Tensor):
    if x.dim() == 2:
        return 1, x.shape[0], x.shape[1]
    if x.dim() == 3:
        return x.shape[0], x.shape[1], x.shape[2]
    raise MxqError("expected a (rows, cols) or (batch, rows, cols) tensor")


# ---- MX quantize / dequantize -----------------------------------------------------------

def mx_quantize(x: torch.Tensor, axes: int, q_row=None, s_row=None, q_col=None, s_col=None,
                stream=None) -> None:
    """x: bf16 (rows, cols) or (batch, rows, cols).  Outputs (uint8, preallocated):
    q_row (b, rows, cols), s_row (b, rows, cols/32), q_col (b, cols, rows),
    s_col (b, cols, rows/32)."""
    batch, rows, cols = _bsc(x)
    px = _dev(x, torch.bfloat16, "x")
    n = batch * rows * cols
    pr = sr = pc = sc = None
    if axes & ROW:
        pr = _dev(q_row, torch.uint8, "q_row", n)
        sr = _dev(s_row, torch.uint8, "s_row", n // 32)
    if axes & COL:
        pc = _dev(q_col, torch.uint8, "q_col", n)
        sc = _dev(s_col, torch.uint8, "s_col", n // 32)
    _check(lib().mx_quantize(px, batch, rows, cols, axes, pr, sr, pc, sc, _stream(stream)))


def mx_dequantize(q: torch.Tensor, s: torch.Tensor, batch: int, rows: int, cols: int,
                  axis: int, y: torch.Tensor, stream=None) -> None:
    n = batch * rows * cols
    pq = _dev(q, torch.uint8, "q", n)
    ps = _dev(s, torch.uint8, "s", n // 32)
    py = _dev(y, torch.bfloat16, "y", n)
    _check(lib().mx_dequantize(pq, ps, batch, rows, cols, axis, py, _stream(stream)))


def empty_mx_outputs(x: torch.Tensor, axes: int):
    """Allocate the uint8 outputs mx_quantize writes for ``x`` (device memory)."""
    batch, rows, cols = _bsc(x)
    kw = dict(dtype=torch.uint8, device=x.device)
    out = {}
    if axes & ROW:
        out["q_row"] = torch.empty((batch, rows, cols), **kw)
        out["s_row"] = torch.empty((batch, rows, cols // 32), **kw)
    if axes & COL:
        out["q_col"] = torch.empty((batch, cols, rows), **kw)
        out["s_col"] = torch.empty((batch, cols, rows // 32), **kw)
    return out


# ---- per-group rowwise --------------------------------------------------------------------

def fp8_per_group_rowwise_quant(x: torch.Tensor, offs: torch.Tensor, out_layout: int,
                                q: torch.Tensor, scales: torch.Tensor, stream=None) -> None:
    """x: bf16 (M, K); offs: int32 (G,) end offsets on the device; q: uint8 (M, K) for
    ROW_MAJOR or (K, M) for COL_MAJOR; scales: fp32 (G, K)."""
    if x.dim() != 2:
        raise MxqError("x must be (M, K)")
    M, K = x.shape
    G = offs.numel()
    px = _dev(x, torch.bfloat16, "x")
    po = _dev(offs, torch.int32, "offs")
    pq = _dev(q, torch.uint8, "q", M * K)
    ps = _dev(scales, torch.float32, "scales", G * K)
    _check(lib().fp8_per_group_rowwise_quant(px, M, K, po, G, out_layout, pq, ps, _stream(stream)))


def fp8_per_group_rowwise_quant_batched(x: torch.Tensor, out_layout: int, q: torch.Tensor, scales: torch.Tensor,
                                        stream=None) -> None:
    """x: bf16 (E, M, K), every matrix its own group; q: uint8 (E, M, K) for ROW_MAJOR or
    (E, K, M) for COL_MAJOR; scales: fp32 (E, K)."""
    if x.dim() != 3:
        raise MxqError("x must be (E, M, K)")
    E, M, K = x.shape
    px = _dev(x, torch.bfloat16, "x")
    pq = _dev(q, torch.uint8, "q", E * M * K)
    ps = _dev(scales, torch.float32, "scales", E * K)
    _check(lib().fp8_per_group_rowwise_quant_batched(px, E, M, K, out_layout, pq, ps, _stream(stream)))


def mx_e4m3_encode_f32(x: torch.Tensor, q: torch.Tensor, stream=None) -> None:
    """fp32 -> E4M3 with the convert every kernel uses (RNE, saturating to 448)."""
    n = x.numel()
    px = _dev(x, torch.float32, "x")
    pq = _dev(q, torch.uint8, "q", n)
    _check(lib().mx_e4m3_encode_f32(px, n, pq, _stream(stream)))


PLAN_KERNELS = {0: "none", 1: "tile", 2: "pair", 3: "stream"}


def fp8_per_group_rowwise_plan(M: int, K: int, G: int, out_layout: int, n_sm: int = 0) -> dict:
    """The kernel and tile shape fp8_per_group_rowwise_quant launches for these sizes
    (host only).  Returns {kernel, slab_cols, cluster, tile_rows, threads}."""
    vals = [ctypes.c_int(0) for _ in range(5)]
    _check(lib().fp8_per_group_rowwise_plan(M, K, G, out_layout, n_sm, *[ctypes.byref(v) for v in vals]))
    kernel, w, cl, rows, threads = (v.value for v in vals)
    return {"kernel": PLAN_KERNELS[kernel], "slab_cols": w, "cluster": cl, "tile_rows": rows, "threads": threads}


WAIT_LIMIT_DEFAULT_NS = 2_000_000_000


def mxq_wait_timeouts() -> int:
    """Number of kernel CTAs that gave up a bounded wait since the library was loaded
    (0 in a healthy run).  Synchronizes the device."""
    n = ctypes.c_uint(0)
    _check(lib().mxq_wait_timeouts(ctypes.byref(n)))
    return n.value


def mxq_wait_abandoned() -> int:
    """Of those, the CTAs whose copies in flight did not land after giving up either
    (0 in a healthy run).  Synchronizes the device."""
    n = ctypes.c_uint(0)
    _check(lib().mxq_wait_abandoned(ctypes.byref(n)))
    return n.value


def mxq_set_wait_limit_ns(ns: int) -> None:
    """Limit of the per-group kernels' bounded waits for later launches (0: give up at
    once, to exercise the give-up path)."""
    _check(lib().mxq_set_wait_limit_ns(int(ns)))


# ---- layouts for the scaled grouped GEMM ---------------------------------------------------

def mxq_transpose_u8(src: torch.Tensor, dst: torch.Tensor, stream=None) -> None:
    """uint8 (rows, cols) or (batch, rows, cols) -> dst (.., cols, rows)."""
    batch, rows, cols = _bsc(src)
    ps = _dev(src, torch.uint8, "src")
    pd = _dev(dst, torch.uint8, "dst", batch * rows * cols)
    _check(lib().mxq_transpose_u8(ps, batch, rows, cols, pd, _stream(stream)))


def mx_scales_blocked_bytes(batch: int, rows: int, n_k: int, G: int = 0) -> int:
    n = int(lib().mx_scales_blocked_bytes(batch, rows, n_k, G))
    if n < 0:
        raise MxqError("invalid sizes for the blocked scale layout")
    return n


def mx_scales_to_blocked(s: torch.Tensor, out: torch.Tensor, offs: torch.Tensor | None = None,
                         stream=None) -> None:
    """E8M0 scales uint8 (rows, n_k) or (batch, rows, n_k) -> out (flat uint8 of
    mx_scales_blocked_bytes), tiled for the block-scaled MMA; with offs (int32 end
    offsets on the device) every group's rows padded to whole 128-row tiles."""
    batch, rows, n_k = _bsc(s)
    G = 0 if offs is None else offs.numel()
    ps = _dev(s, torch.uint8, "s")
    po = None if offs is None else _dev(offs, torch.int32, "offs")
    pout = _dev(out, torch.uint8, "out")
    if out.numel() < mx_scales_blocked_bytes(batch, rows, n_k, G):
        raise MxqError("out is smaller than mx_scales_blocked_bytes")
    _check(lib().mx_scales_to_blocked(ps, batch, rows, n_k, po, G, pout, _stream(stream)))


# ---- MXFP8 grouped GEMM -------------------------------------------------------------------------

def mx_grouped_gemm(qa: torch.Tensor, sfa_blocked: torch.Tensor, qb: torch.Tensor, sfb_blocked: torch.Tensor,
                    offs: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    """qa uint8 (M, K) E4M3 tokens; sfa_blocked: their scales from mx_scales_to_blocked
    with offs; qb uint8 (G, N, K) expert weights; sfb_blocked: their scales from
    mx_scales_to_blocked (per matrix); offs int32 (G,) end offsets; out bf16 (M, N)."""
    if qa.dim() != 2 or qb.dim() != 3:
        raise MxqError("qa must be (M, K) and qb (G, N, K)")
    M, K = qa.shape
    G, N, K2 = qb.shape
    if K2 != K or offs.numel() != G:
        raise MxqError("qa, qb and offs disagree on K or G")
    pa = _dev(qa, torch.uint8, "qa")
    pb = _dev(qb, torch.uint8, "qb")
    psa = _dev(sfa_blocked, torch.uint8, "sfa_blocked")
    psb = _dev(sfb_blocked, torch.uint8, "sfb_blocked")
    if sfa_blocked.numel() < mx_scales_blocked_bytes(1, M, K // 32, G):
        raise MxqError("sfa_blocked is smaller than mx_scales_blocked_bytes(1, M, K/32, G)")
    if sfb_blocked.numel() < mx_scales_blocked_bytes(G, N, K // 32, 0):
        raise MxqError("sfb_blocked is smaller than mx_scales_blocked_bytes(G, N, K/32, 0)")
    po = _dev(offs, torch.int32, "offs")
    pout = _dev(out, torch.bfloat16, "out", M * N)
    _check(lib().mx_grouped_gemm(pa, psa, pb, psb, po, G, M, N, K, pout, _stream(stream)))
