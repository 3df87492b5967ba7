"""GPU parity at the full workload sizes, in the launch configuration the benchmark uses.

The CUDA path runs on the whole tensors and EVERY output byte, scale and dequantized
value is compared with the oracle, bit for bit.  The oracle works on independent
slabs (row slabs for MX blocks, column slabs for per-group features) in a spawned
process pool, always from the seeded inputs, never from a GPU result.  The outputs
come from canary-filled buffers, so a byte the kernels should have written but did
not shows up too.
"""
import numpy as np
import pytest
import torch

import oracle
import mxfp8_quantization_moe_mx_b200 as mxq
from mxfp8_quantization_moe_mx_b200 import workloads as wl

import _oracle_slabs as slabs
from _gpu import CANARY, bits_of, ensure_lib, same_f32

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ensure_lib()
    before = mxq.mxq_wait_timeouts()
    yield
    # no tile copy of the full-size runs ran out of its bounded wait
    assert mxq.mxq_wait_timeouts() == before


@pytest.fixture(scope="module")
def pool():
    p = slabs.make_pool()
    yield p
    p.shutdown()


def _filled(shape, dtype=torch.uint8, fill=CANARY):
    return torch.full(shape, fill, dtype=dtype, device="cuda")


def _mx_outputs(batch, rows, cols, axes):
    out = {}
    if axes & mxq.ROW:
        out["q_row"] = _filled((batch, rows, cols))
        out["s_row"] = _filled((batch, rows, cols // 32))
    if axes & mxq.COL:
        out["q_col"] = _filled((batch, cols, rows))
        out["s_col"] = _filled((batch, cols, rows // 32))
    return out


def _assert_mx(got: dict, ref: dict, what: str):
    for k, r in ref.items():
        if k == "y":
            continue
        g = got[k]
        g = g.cpu().numpy() if isinstance(g, torch.Tensor) else g
        assert g.shape == r.shape, (what, k, g.shape, r.shape)
        np.testing.assert_array_equal(g, r, err_msg=f"{what}: {k}")


def _assert_per_group(q_gpu, s_gpu, layout, q_ref, s_ref, what):
    """q_ref is row-major (M, K); a column-major GPU result is compared as its transpose."""
    q = q_gpu.cpu().numpy()
    if layout == mxq.COL_MAJOR:
        q = q.T
    assert same_f32(s_gpu.cpu().numpy(), s_ref), f"{what}: scales"
    if not np.array_equal(q, q_ref):
        bad = np.argwhere(q != q_ref)
        raise AssertionError(f"{what}: {len(bad)} codes differ, first at (row, col) {bad[0].tolist()}")


# ---- dispatch payload (65536 x 5120): the benchmark step --------------------------------------

def test_dispatch_payload_step(pool):
    """MX dual-axis quantize -> MX dequantize -> per-group (16 experts, row-major) on
    the (65536, 5120) dispatch payload, exactly the calls the benchmark times.  The
    oracle chains the same three steps on its own results."""
    t = wl.dispatch()
    x, offs = t["x"], t["offs"].numpy()
    xb = bits_of(x)
    M, K = x.shape
    assert offs[-1] == M
    futs = [(a, b, pool.submit(slabs.mx_round_trip_slab, np.ascontiguousarray(xb[a:b])))
            for a, b in slabs.row_edges(M, 4096)]

    xd = x.cuda()
    out = _mx_outputs(1, M, K, mxq.ROW | mxq.COL)
    mxq.mx_quantize(xd, mxq.ROW | mxq.COL, **out)
    y = torch.full((M, K), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    mxq.mx_dequantize(out["q_row"], out["s_row"], 1, M, K, mxq.ROW, y)
    q = _filled((M, K))
    s = torch.full((offs.size, K), float("nan"), device="cuda")
    mxq.fp8_per_group_rowwise_quant(y, torch.from_numpy(offs).cuda(), mxq.ROW_MAJOR, q, s)
    torch.cuda.synchronize()
    del xd

    ref = {"q_row": np.empty((M, K), np.uint8), "s_row": np.empty((M, K // 32), np.uint8),
           "q_col": np.empty((K, M), np.uint8), "s_col": np.empty((K, M // 32), np.uint8)}
    y_ref = np.empty((M, K), np.uint16)
    for a, b, f in futs:
        r = f.result()
        ref["q_row"][a:b], ref["s_row"][a:b] = r["q_row"], r["s_row"]
        ref["q_col"][:, a:b], ref["s_col"][:, a // 32:b // 32] = r["q_col"], r["s_col"]
        y_ref[a:b] = r["y"]
    got = {k: v[0] for k, v in out.items()}
    _assert_mx(got, ref, "dispatch dual-axis quantize")
    del got, out, ref
    np.testing.assert_array_equal(bits_of(y), y_ref, err_msg="dispatch dequantize")
    del y
    q_ref, s_ref = slabs.per_group_whole(pool, y_ref, offs)
    _assert_per_group(q, s, mxq.ROW_MAJOR, q_ref, s_ref, "dispatch per-group (16 experts)")


# ---- per-group rowwise at (16640, 5120), 16..128 groups, both layouts --------------------------

@pytest.mark.parametrize("G", [16, 32, 64, 128])
def test_per_group_config(pool, G):
    t = wl.per_group(n_groups=G)
    x, offs = t["x"], t["offs"].numpy()
    M, K = x.shape
    assert offs[-1] == M
    xb = bits_of(x)
    q_ref, s_ref = slabs.per_group_whole(pool, xb, offs)
    xd, od = x.cuda(), torch.from_numpy(offs).cuda()
    for layout in (mxq.ROW_MAJOR, mxq.COL_MAJOR):
        q = _filled((M, K) if layout == mxq.ROW_MAJOR else (K, M))
        s = torch.full((G, K), float("nan"), device="cuda")
        mxq.fp8_per_group_rowwise_quant(xd, od, layout, q, s)
        torch.cuda.synchronize()
        _assert_per_group(q, s, layout, q_ref, s_ref, f"per-group (16640, 5120) G={G} layout={layout}")
        if layout == mxq.COL_MAJOR:
            # the pages' route for many groups: column-major codes, then the transform
            qt = _filled((M, K))
            mxq.mxq_transpose_u8(q, qt)
            torch.cuda.synchronize()
            _assert_per_group(qt, s, mxq.ROW_MAJOR, q_ref, s_ref, f"transformed column-major codes G={G}")


# ---- dual-axis MXFP8 for the backward pass ------------------------------------------------------

def test_dual_axis_activations(pool):
    x = wl.dual_axis(experts=1, hidden=32)["act"]
    M, K = x.shape
    ref = slabs.mx_quantize_whole(pool, bits_of(x), mxq.ROW | mxq.COL)
    out = _mx_outputs(1, M, K, mxq.ROW | mxq.COL)
    mxq.mx_quantize(x.cuda(), mxq.ROW | mxq.COL, **out)
    torch.cuda.synchronize()
    _assert_mx({k: v[0] for k, v in out.items()}, ref, "activations (16384, 5120)")


def test_dual_axis_expert_weights(pool):
    """(16, 8192, 5120) in one batched call, every expert compared whole."""
    w = wl.dual_axis()["w"]
    B, R, C = w.shape
    wb = bits_of(w)
    futs = [pool.submit(slabs.mx_quantize_slab, np.ascontiguousarray(wb[e]), mxq.ROW | mxq.COL) for e in range(B)]
    out = _mx_outputs(B, R, C, mxq.ROW | mxq.COL)
    mxq.mx_quantize(w.cuda(), mxq.ROW | mxq.COL, **out)
    torch.cuda.synchronize()
    host = {k: v.cpu().numpy() for k, v in out.items()}
    for e, f in enumerate(futs):
        _assert_mx({k: v[e] for k, v in host.items()}, f.result(), f"expert weights, expert {e}")


# ---- stress mix ----------------------------------------------------------------------------------

@pytest.fixture(scope="module")
def stress_inputs():
    t = wl.stress()
    return t["x"], t["offs"].numpy()


def test_stress_per_group(pool, stress_inputs):
    """(131072, 5120), 128 Zipf(1.2) groups with 20 empty, column-major output."""
    x, offs = stress_inputs
    M, K = x.shape
    assert offs[-1] == M
    q_ref, s_ref = slabs.per_group_whole(pool, bits_of(x), offs, n_slabs=64)
    q = _filled((K, M))
    s = torch.full((offs.size, K), float("nan"), device="cuda")
    mxq.fp8_per_group_rowwise_quant(x.cuda(), torch.from_numpy(offs).cuda(), mxq.COL_MAJOR, q, s)
    torch.cuda.synchronize()
    _assert_per_group(q, s, mxq.COL_MAJOR, q_ref, s_ref, "stress per-group")


def test_stress_mx(pool, stress_inputs):
    x, _ = stress_inputs
    M, K = x.shape
    ref = slabs.mx_quantize_whole(pool, bits_of(x), mxq.ROW | mxq.COL)
    out = _mx_outputs(1, M, K, mxq.ROW | mxq.COL)
    mxq.mx_quantize(x.cuda(), mxq.ROW | mxq.COL, **out)
    torch.cuda.synchronize()
    _assert_mx({k: v[0] for k, v in out.items()}, ref, "stress MX dual-axis")
