"""GPU parity at the full workload sizes, in the launch configuration the benchmark uses.

The CUDA path runs on the whole tensors; the oracle recomputes sampled pieces that it
can compute on their own -- whole rows (1x32 blocks), whole 32-row bands (32x1
blocks), whole features (per-group: every row of the sampled columns) -- always from
the seeded inputs, never from a GPU result.  Comparisons are bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
import mxfp8_quantization_moe_mx_b200 as mxq
from mxfp8_quantization_moe_mx_b200 import workloads as wl

from _gpu import bits_of, ensure_lib, same_f32

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ensure_lib()


def _rows_sample(n, k, seed):
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(n, size=k, replace=False))


def _check_rows(xb, q_row, s_row, rows):
    """Compare sampled rows of a 1x32 quantization (q_row/s_row as device tensors)."""
    ref = oracle.mx_quantize(np.ascontiguousarray(xb[rows]), oracle.ROW)
    idx = torch.as_tensor(rows, device=q_row.device)
    np.testing.assert_array_equal(q_row.index_select(0, idx).cpu().numpy(), ref["q_row"])
    np.testing.assert_array_equal(s_row.index_select(0, idx).cpu().numpy(), ref["s_row"])
    return ref


def _check_bands(xb, q_col, s_col, bands):
    """Compare sampled 32-row bands of a 32x1 quantization; xb (rows, cols),
    q_col (cols, rows), s_col (cols, rows/32)."""
    for b in bands:
        ref = oracle.mx_quantize(np.ascontiguousarray(xb[32 * b:32 * b + 32]), oracle.COL)
        np.testing.assert_array_equal(q_col[:, 32 * b:32 * b + 32].cpu().numpy(), ref["q_col"])
        np.testing.assert_array_equal(s_col[:, b:b + 1].cpu().numpy(), ref["s_col"])


def _check_features(xb, offs, layout, q, s, feats):
    """Per-group: every row of the sampled features (feature groups of 8 columns)."""
    cols = np.concatenate([np.arange(8 * f, 8 * f + 8) for f in feats])
    sub = np.ascontiguousarray(xb[:, cols])
    qr, sr = oracle.per_group_quant(sub, offs, layout)
    idx = torch.as_tensor(cols, device=q.device)
    if layout == mxq.ROW_MAJOR:
        got = q.index_select(1, idx).cpu().numpy()
        rows_in_groups = int(min(max(0, int(np.max(offs))), xb.shape[0]))
        np.testing.assert_array_equal(got[:rows_in_groups], qr[:rows_in_groups])
    else:
        got = q.index_select(0, idx).cpu().numpy()
        rows_in_groups = int(min(max(0, int(np.max(offs))), xb.shape[0]))
        np.testing.assert_array_equal(got[:, :rows_in_groups], qr[:, :rows_in_groups])
    assert same_f32(s.index_select(1, idx).cpu().numpy(), sr)


# ---- dispatch payload (65536 x 5120): the benchmark step --------------------------------------

def test_dispatch_payload_step():
    """MX dual-axis quantize -> MX dequantize -> per-group (16 experts, row-major) on
    the (65536, 5120) dispatch payload, exactly the calls the benchmark times."""
    t = wl.dispatch()
    x, offs = t["x"], t["offs"]
    xb = bits_of(x)
    M, K = x.shape
    xd = x.cuda()
    out = mxq.empty_mx_outputs(xd, mxq.ROW | mxq.COL)
    mxq.mx_quantize(xd, mxq.ROW | mxq.COL, **out)
    y = torch.empty_like(xd)
    mxq.mx_dequantize(out["q_row"], out["s_row"], 1, M, K, mxq.ROW, y)
    od = offs.cuda()
    q = torch.empty(M, K, dtype=torch.uint8, device="cuda")
    s = torch.empty(offs.numel(), K, dtype=torch.float32, device="cuda")
    mxq.fp8_per_group_rowwise_quant(y, od, mxq.ROW_MAJOR, q, s)
    torch.cuda.synchronize()

    rows = _rows_sample(M, 256, 1)
    ref = _check_rows(xb, out["q_row"][0], out["s_row"][0], rows)
    _check_bands(xb, out["q_col"][0], out["s_col"][0], _rows_sample(M // 32, 24, 2))
    # dequant: oracle dequant of the oracle's own quantized rows
    yref = oracle.mx_dequantize(ref["q_row"], ref["s_row"], 1, len(rows), K, oracle.ROW)
    np.testing.assert_array_equal(bits_of(y.index_select(0, torch.as_tensor(rows, device="cuda")).cpu()), yref)
    # per-group on the dequantized tokens: the oracle rebuilds those tokens for the
    # sampled 32-column blocks from the seeded input, then scales them per group
    rng = np.random.default_rng(3)
    blocks = np.sort(rng.choice(K // 32, size=3, replace=False))
    cols = np.concatenate([np.arange(32 * b, 32 * b + 32) for b in blocks])
    sub = np.ascontiguousarray(xb[:, cols])
    rq = oracle.mx_quantize(sub, oracle.ROW)
    ysub = oracle.mx_dequantize(rq["q_row"], rq["s_row"], 1, M, len(cols), oracle.ROW)
    qr, sr = oracle.per_group_quant(ysub, offs.numpy(), oracle.ROW_MAJOR)
    idx = torch.as_tensor(cols, device="cuda")
    np.testing.assert_array_equal(q.index_select(1, idx).cpu().numpy(), qr)
    assert same_f32(s.index_select(1, idx).cpu().numpy(), sr)


# ---- per-group rowwise at (16640, 5120), 16..128 groups ----------------------------------------

@pytest.fixture(scope="module")
def per_group_inputs():
    return {G: wl.per_group(n_groups=G) for G in (16, 32, 64, 128)}


@pytest.mark.parametrize("G", [16, 32, 64, 128])
@pytest.mark.parametrize("layout", [0, 1])
def test_per_group_config(per_group_inputs, G, layout):
    t = per_group_inputs[G]
    x, offs = t["x"], t["offs"]
    M, K = x.shape
    xd = x.cuda()
    shape = (M, K) if layout == mxq.ROW_MAJOR else (K, M)
    q = torch.empty(shape, dtype=torch.uint8, device="cuda")
    s = torch.empty(G, K, dtype=torch.float32, device="cuda")
    mxq.fp8_per_group_rowwise_quant(xd, offs.cuda(), layout, q, s)
    torch.cuda.synchronize()
    feats = _rows_sample(K // 8, 6, G + layout)
    _check_features(bits_of(x), offs.numpy(), layout, q, s, feats)


# ---- dual-axis MXFP8 for the backward pass ------------------------------------------------------

def test_dual_axis_config():
    t = wl.dual_axis()
    for name in ("act", "w"):
        x = t[name]
        xb = bits_of(x)
        xd = x.cuda()
        out = mxq.empty_mx_outputs(xd, mxq.ROW | mxq.COL)
        mxq.mx_quantize(xd, mxq.ROW | mxq.COL, **out)
        torch.cuda.synchronize()
        if x.dim() == 2:
            xb = xb[None]
        B, R, C = xb.shape
        for e in sorted(set([0, B - 1, B // 2])):
            _check_rows(xb[e], out["q_row"][e], out["s_row"][e], _rows_sample(R, 64, e + 10))
            _check_bands(xb[e], out["q_col"][e], out["s_col"][e], _rows_sample(R // 32, 6, e + 20))


# ---- stress mix ----------------------------------------------------------------------------------

def test_stress_config():
    t = wl.stress()
    x, offs = t["x"], t["offs"]
    xb = bits_of(x)
    M, K = x.shape
    xd = x.cuda()
    q = torch.empty(K, M, dtype=torch.uint8, device="cuda")
    s = torch.empty(offs.numel(), K, dtype=torch.float32, device="cuda")
    mxq.fp8_per_group_rowwise_quant(xd, offs.cuda(), mxq.COL_MAJOR, q, s)
    torch.cuda.synchronize()
    _check_features(xb, offs.numpy(), mxq.COL_MAJOR, q, s, _rows_sample(K // 8, 6, 4))
    del q
    out = mxq.empty_mx_outputs(xd, mxq.ROW | mxq.COL)
    mxq.mx_quantize(xd, mxq.ROW | mxq.COL, **out)
    torch.cuda.synchronize()
    _check_rows(xb, out["q_row"][0], out["s_row"][0], _rows_sample(M, 128, 5))
    _check_bands(xb, out["q_col"][0], out["s_col"][0], _rows_sample(M // 32, 8, 6))
