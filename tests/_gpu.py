"""Helpers for the GPU parity tests: run the CUDA path through the C ABI (via the thin
binding) on CPU tensors and bring the results back as numpy arrays."""
import numpy as np
import torch

import mxfp8_quantization_moe_mx_b200 as mxq
from mxfp8_quantization_moe_mx_b200 import build as mxq_build

CANARY = 0xA5


def ensure_lib():
    mxq_build.build()
    mxq.lib()


def bits_of(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def gpu_mx_quantize(x: torch.Tensor, axes: int, guard: int = 64):
    """x: CPU or CUDA bf16 (rows, cols) or (batch, rows, cols).  Outputs are carved
    out of larger canary-filled buffers and the guard bytes are checked afterwards."""
    xd = x.cuda() if not x.is_cuda else x
    batch, rows, cols = (1, *xd.shape) if xd.dim() == 2 else tuple(xd.shape)
    n = batch * rows * cols
    bufs, views = {}, {}
    shapes = {}
    if axes & mxq.ROW:
        shapes["q_row"] = (batch, rows, cols)
        shapes["s_row"] = (batch, rows, cols // 32)
    if axes & mxq.COL:
        shapes["q_col"] = (batch, cols, rows)
        shapes["s_col"] = (batch, cols, rows // 32)
    for k, shp in shapes.items():
        size = int(np.prod(shp))
        b = torch.full((size + 2 * guard,), CANARY, dtype=torch.uint8, device="cuda")
        bufs[k] = b
        views[k] = b[guard:guard + size].view(shp)
    mxq.mx_quantize(xd, axes, **views)
    torch.cuda.synchronize()
    out = {}
    for k, b in bufs.items():
        h = b.cpu().numpy()
        assert np.all(h[:guard] == CANARY) and np.all(h[-guard:] == CANARY), f"{k}: guard bytes overwritten"
        out[k] = h[guard:-guard].reshape(shapes[k])
        if batch == 1 and xd.dim() == 2:
            out[k] = out[k][0]
    return out


def gpu_mx_dequantize(q: np.ndarray, s: np.ndarray, batch: int, rows: int, cols: int, axis: int,
                      guard: int = 64) -> np.ndarray:
    qd = torch.from_numpy(np.ascontiguousarray(q)).cuda()
    sd = torch.from_numpy(np.ascontiguousarray(s)).cuda()
    n = batch * rows * cols
    buf = torch.full((n + 2 * guard,), -1, dtype=torch.int16, device="cuda")
    y = buf[guard:guard + n].view(torch.bfloat16)
    mxq.mx_dequantize(qd, sd, batch, rows, cols, axis, y)
    torch.cuda.synchronize()
    h = buf.cpu().numpy().view(np.uint16)
    assert np.all(h[:guard] == 0xFFFF) and np.all(h[-guard:] == 0xFFFF), "guard overwritten"
    out = h[guard:-guard].reshape(batch, rows, cols)
    return out[0] if batch == 1 else out


def gpu_per_group(x: torch.Tensor, offs, layout: int, guard: int = 64):
    """Returns (q, scales) as numpy; q keeps CANARY in bytes the kernel must not write."""
    xd = x.cuda() if not x.is_cuda else x
    M, K = xd.shape
    od = torch.as_tensor(np.asarray(offs, dtype=np.int32)).cuda()
    G = od.numel()
    qb = torch.full((M * K + 2 * guard,), CANARY, dtype=torch.uint8, device="cuda")
    sb = torch.full((G * K + 2 * guard,), float("nan"), dtype=torch.float32, device="cuda")
    q = qb[guard:guard + M * K]
    s = sb[guard:guard + G * K]
    mxq.fp8_per_group_rowwise_quant(xd, od, layout, q, s)
    torch.cuda.synchronize()
    qh = qb.cpu().numpy()
    sh = sb.cpu().numpy()
    assert np.all(qh[:guard] == CANARY) and np.all(qh[-guard:] == CANARY), "q guard overwritten"
    assert np.all(np.isnan(sh[:guard])) and np.all(np.isnan(sh[-guard:])), "scale guard overwritten"
    shape = (M, K) if layout == mxq.ROW_MAJOR else (K, M)
    return qh[guard:-guard].reshape(shape), sh[guard:-guard].reshape(G, K)


def same_f32(a: np.ndarray, b: np.ndarray) -> bool:
    """Bitwise equality of fp32 arrays."""
    return np.array_equal(np.ascontiguousarray(a, np.float32).view(np.uint32),
                          np.ascontiguousarray(b, np.float32).view(np.uint32))
