"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle, bit for bit.

Tolerance is zero everywhere: E4M3 bytes, E8M0 bytes, fp32 scales (bitwise) and
dequantized bf16 (bitwise).  Small cases compare every output; the full-size
workloads (the shapes the benchmark runs, same launch configuration) compare sampled
rows / bands / features, which the oracle computes independently of the rest.
Output buffers are carved from canary-filled allocations and the guard bytes around
them are checked after every call.
"""
import numpy as np
import pytest
import torch

import oracle
import mxfp8_quantization_moe_mx_b200 as mxq
from mxfp8_quantization_moe_mx_b200 import workloads as wl

from _gpu import CANARY, bits_of, ensure_lib, gpu_mx_dequantize, gpu_mx_quantize, gpu_per_group, same_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ensure_lib()


def mixed(batch, rows, cols, seed=7):
    """A stress-mix tensor (normals, subnormals, +-448, values above 448, zero blocks)."""
    x = wl.stress(seed=seed, M=batch * rows, K=cols, n_groups=4, n_empty=1)["x"]
    return x.view(batch, rows, cols) if batch > 1 else x.view(rows, cols)


def assert_mx_equal(got, ref, keys):
    for k in keys:
        np.testing.assert_array_equal(got[k], ref[k], err_msg=k)


# ---- tiny configuration: every op, every output --------------------------------------------

def test_tiny_config_all_ops():
    t = wl.tiny()
    x, offs = t["x"], t["offs"].numpy()
    xb = bits_of(x)
    for axes in (mxq.ROW, mxq.COL, mxq.ROW | mxq.COL):
        got = gpu_mx_quantize(x, axes)
        ref = oracle.mx_quantize(xb, axes)
        assert_mx_equal(got, ref, ref.keys())
    r = oracle.mx_quantize(xb, mxq.ROW | mxq.COL)
    y = gpu_mx_dequantize(r["q_row"], r["s_row"], 1, 256, 512, mxq.ROW)
    np.testing.assert_array_equal(y, oracle.mx_dequantize(r["q_row"], r["s_row"], 1, 256, 512, 1))
    yc = gpu_mx_dequantize(r["q_col"], r["s_col"], 1, 256, 512, mxq.COL)
    np.testing.assert_array_equal(yc, oracle.mx_dequantize(r["q_col"], r["s_col"], 1, 256, 512, 2))
    for layout in (mxq.ROW_MAJOR, mxq.COL_MAJOR):
        q, s = gpu_per_group(x, offs, layout)
        shape = (256, 512) if layout == mxq.ROW_MAJOR else (512, 256)
        qr, sr = oracle.per_group_quant(xb, offs, layout, q_init=np.full(shape, CANARY))
        assert same_f32(s, sr)
        np.testing.assert_array_equal(q, qr)


# ---- MX quantize / dequantize over shapes with ragged tiles --------------------------------

MX_SHAPES = [(1, 32, 32), (1, 320, 96), (3, 96, 160), (2, 288, 64), (1, 1024, 2048), (4, 64, 32),
             (2, 512, 128)]


@pytest.mark.parametrize("shape", MX_SHAPES)
@pytest.mark.parametrize("axes", [1, 2, 3])
def test_mx_quantize_shapes(shape, axes):
    b, r, c = shape
    x = mixed(b, r, c, seed=11 + r + c)
    got = gpu_mx_quantize(x, axes)
    ref = oracle.mx_quantize(bits_of(x), axes)
    assert_mx_equal(got, ref, ref.keys())


@pytest.mark.parametrize("shape", MX_SHAPES)
@pytest.mark.parametrize("axis", [1, 2])
def test_mx_dequantize_shapes(shape, axis):
    b, r, c = shape
    rng = np.random.default_rng(r * c + axis)
    n = b * r * c
    q = rng.integers(0, 256, size=n, dtype=np.uint8)
    s = rng.integers(0, 256, size=n // 32, dtype=np.uint8)  # includes 0 (2^-127) and 0xFF (NaN)
    y = gpu_mx_dequantize(q, s, b, r, c, axis)
    ref = oracle.mx_dequantize(q, s, b, r, c, axis)
    np.testing.assert_array_equal(y, ref)


def test_mx_quantize_many_tiles_per_cta():
    """Many more 256 x 64 tiles than resident CTAs (several waves, each CTA prefetching
    a later tile into L2), checked in full."""
    x = mixed(1, 4096, 8192, seed=77)
    got = gpu_mx_quantize(x, 3)
    ref = oracle.mx_quantize(bits_of(x), 3)
    assert_mx_equal(got, ref, ref.keys())


def test_mx_grid_split_over_matrices():
    """More matrices than the grid's z limit (65535): the tile kernels go out as two
    launches; every output of every matrix checked."""
    b, r, c = 65537, 32, 32
    x = (torch.randn(b, r, c, device="cuda") * 3).to(torch.bfloat16)
    xb = bits_of(x)
    got = gpu_mx_quantize(x, mxq.ROW | mxq.COL)
    ref = oracle.mx_quantize(xb, mxq.ROW | mxq.COL)
    assert_mx_equal(got, ref, ref.keys())
    y = gpu_mx_dequantize(ref["q_col"], ref["s_col"], b, r, c, mxq.COL)
    np.testing.assert_array_equal(y, oracle.mx_dequantize(ref["q_col"], ref["s_col"], b, r, c, 2))


def test_mx_grid_split_over_row_tiles():
    """More 256-row tiles than the grid's y limit (65535 x 256 rows, 32 columns): the
    tile kernels go out as two launches.  Checked on the first tile, the tiles around the
    split and the last one (column blocks stay within their 32-row bands, so a band range
    is checked against the oracle run on those rows alone)."""
    rows, cols = 65536 * 256 + 256, 32
    x = (torch.randn(rows, cols, device="cuda") * 5).to(torch.bfloat16)
    out = mxq.empty_mx_outputs(x, mxq.ROW | mxq.COL)
    mxq.mx_quantize(x, mxq.ROW | mxq.COL, **out)
    y = torch.empty_like(x)
    mxq.mx_dequantize(out["q_col"], out["s_col"], 1, rows, cols, mxq.COL, y)
    torch.cuda.synchronize()
    for r0, r1 in ((0, 512), (65535 * 256 - 512, 65535 * 256 + 256), (rows - 512, rows)):
        xb = bits_of(x[r0:r1])
        ref = oracle.mx_quantize(xb, mxq.ROW | mxq.COL)
        np.testing.assert_array_equal(out["q_row"][0, r0:r1].cpu().numpy(), ref["q_row"])
        np.testing.assert_array_equal(out["s_row"][0, r0:r1].cpu().numpy(), ref["s_row"])
        np.testing.assert_array_equal(out["q_col"][0, :, r0:r1].cpu().numpy(), ref["q_col"])
        np.testing.assert_array_equal(out["s_col"][0, :, r0 // 32:r1 // 32].cpu().numpy(), ref["s_col"])
        yr = oracle.mx_dequantize(ref["q_col"], ref["s_col"], 1, r1 - r0, cols, 2)
        np.testing.assert_array_equal(bits_of(y[r0:r1]), yr)
    del x, y, out
    torch.cuda.empty_cache()


def test_mx_roundtrip_matches_oracle_roundtrip():
    x = mixed(1, 512, 1024, seed=3)
    got = gpu_mx_quantize(x, mxq.ROW | mxq.COL)
    for axis, q, s in ((1, "q_row", "s_row"), (2, "q_col", "s_col")):
        y = gpu_mx_dequantize(got[q], got[s], 1, 512, 1024, axis)
        ref = oracle.mx_dequantize(got[q], got[s], 1, 512, 1024, axis)
        np.testing.assert_array_equal(y, ref)


def test_mx_nonfinite_blocks():
    x = torch.randn(64, 96).to(torch.bfloat16)
    xb = bits_of(x).copy()
    xb[0, 5] = 0x7F80      # +inf in a row block
    xb[3, 40] = 0xFFC1     # NaN
    xb[40, 70] = 0xFF80    # -inf
    xt = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16)
    got = gpu_mx_quantize(xt, mxq.ROW | mxq.COL)
    ref = oracle.mx_quantize(xb, mxq.ROW | mxq.COL)
    assert_mx_equal(got, ref, ref.keys())


# ---- per-group rowwise ------------------------------------------------------------------------

def _per_group_case(M, K, offs, seed):
    x = wl.stress(seed=seed, M=M, K=K if K % 32 == 0 else K + (32 - K % 32), n_groups=3, n_empty=0)["x"]
    x = x[:, :K].contiguous()
    xb = bits_of(x)
    for layout in (mxq.ROW_MAJOR, mxq.COL_MAJOR):
        q, s = gpu_per_group(x, offs, layout)
        shape = (M, K) if layout == mxq.ROW_MAJOR else (K, M)
        qr, sr = oracle.per_group_quant(xb, offs, layout, q_init=np.full(shape, CANARY))
        assert same_f32(s, sr), (M, K, layout)
        np.testing.assert_array_equal(q, qr, err_msg=f"M={M} K={K} layout={layout}")


@pytest.mark.parametrize("M,K,offs", [
    (256, 64, [64, 64, 200, 256]),                 # empty group, exact cover
    (1000, 72, [100, 350, 351, 900]),              # K not a multiple of 64, trailing rows
    (1001, 136, [7, 13, 500, 1001]),               # M not a multiple of 8, odd starts
    (333, 8, [333]),                               # one group, one vector of features
    (512, 128, [0, 0, 512, 512]),                  # leading and trailing empty groups
    (600, 64, [300, 100, 700, -5, 450]),           # malformed: decreasing, past M, negative
    (40, 64, [2 ** 31 - 1]),                       # offset far past M
])
def test_per_group_edge_cases(M, K, offs):
    _per_group_case(M, K, offs, seed=M + K)


@pytest.mark.parametrize("M,K,G", [(2048, 320, 1), (4096, 192, 3), (6000, 128, 16),
                                    (5000, 64, 128), (3000, 200, 130)])
def test_per_group_uniform_groups(M, K, G):
    g = torch.Generator().manual_seed(M + G)
    offs = wl.uniform_group_offsets(g, M, G).numpy()
    _per_group_case(M, K, offs, seed=G)


def test_per_group_skew_exceeds_on_chip_capacity():
    # average group tiny (CS = 1, no staging) but one group of 6000 rows: re-read path
    M, G = 7000, 64
    sizes = np.full(G, 1000 // 63)
    sizes[17] = 0
    sizes[5] = M - sizes.sum() + sizes[5]
    offs = np.cumsum(sizes).astype(np.int32)
    assert offs[-1] == M and sizes.max() > 5000
    _per_group_case(M, 128, offs, seed=5)


def test_per_group_large_groups_use_clusters():
    # 4096-row groups: clusters of 8 CTAs with two staged steps each
    M, G = 32768, 8
    offs = (np.arange(1, G + 1) * (M // G)).astype(np.int32)
    offs[2] += 13  # shift one boundary off the 8-row grid
    _per_group_case(M, 64, offs, seed=9)


@pytest.mark.parametrize("M,K,sizes", [
    # 64-column tiles (TMA boxes of 32 rows): sizes around one and two boxes
    (513, 136, [32, 33, 31, 64, 65, 1, 0, 96, 191]),
    # 32-column tiles (boxes of 64 rows): sizes around the box, odd tails, overflow
    (3000, 72, [64, 65, 63, 127, 128, 129, 3, 2421]),
    # medium groups, M not a multiple of 8 (column-major byte path), one group past r_cap
    (9001, 136, [700, 750, 800, 751, 749, 2600, 1, 0, 900, 650, 600, 100]),
    # ~1000-row groups, M a multiple of 8: 32-column tiles over pairs of CTAs for
    # column-major output (rotated octets), starts off the 8-row grid, a group twice
    # its tile, a partial last slab
    (12288, 200, [1000, 999, 1001, 1003, 997, 1, 0, 1100, 900, 1024, 33, 3230]),
    # ~1400-row groups: 16-column single-CTA tiles for column-major output
    (16800, 96, [1401, 1399, 1393, 1407, 1, 1410, 1389, 1402, 0, 1398, 1404, 2796]),
])
def test_per_group_tile_box_edges(M, K, sizes):
    offs = np.cumsum(np.asarray(sizes)).astype(np.int32)
    assert offs[-1] <= M
    _per_group_case(M, K, offs, seed=len(sizes) + K)


@pytest.mark.parametrize("M,K,sizes", [
    # large groups: tiles split across thread-block clusters; groups larger than the
    # cluster's tiles (extra rows through global memory), an empty and a 3-row group,
    # M not a multiple of 8
    (20001, 136, [5000, 0, 7000, 3, 7998]),
    # exact cover with split points on and off the 32-row grid
    (16384, 64, [4096, 4096 + 33, 4096 - 33, 4096]),
    # ~5000-row average: 32-column tiles over 8-CTA clusters in both layouts (groups
    # above the cluster's resident rows take the global-memory path), an empty and a
    # 13-row group, a partial last slab, M not a multiple of 8
    (42001, 136, [7000, 6500, 0, 7300, 13, 6900, 7100, 7188]),
])
def test_per_group_cluster_tiles(M, K, sizes):
    offs = np.cumsum(np.asarray(sizes)).astype(np.int32)
    assert offs[-1] <= M
    _per_group_case(M, K, offs, seed=M % 97)


@pytest.mark.parametrize("M,K,sizes", [
    # a skewed split: two groups far larger than their tiles (spread over every SM by the
    # oversized-group kernel), the first group among them, empty groups, odd starts
    (20000, 136, [12000, 0, 37, 300, 4000, 1, 0, 900, 700, 500, 400, 300, 200, 100, 63, 0]),
    # the same with M not a multiple of 8 and the largest group last
    (20001, 72, [5, 300, 0, 1200, 600, 13, 900, 400, 250, 120, 2000, 11, 0, 700, 60, 13440]),
])
def test_per_group_oversized_groups(M, K, sizes):
    offs = np.cumsum(np.asarray(sizes)).astype(np.int32)
    assert offs[-1] <= M
    _per_group_case(M, K, offs, seed=M % 89)


@pytest.mark.parametrize("M,K,sizes", [
    # average group above what eight CTAs of 16..32-column tiles hold: the two-pass
    # streaming kernel (tile kept in L2 between its passes), both layouts
    (49152, 72, [16384, 16384, 16384]),
    # the same with an empty group, uneven sizes and M not a multiple of 8 (byte stores)
    (49153, 136, [20000, 0, 13000, 16153]),
])
def test_per_group_streaming_kernel(M, K, sizes):
    offs = np.cumsum(np.asarray(sizes)).astype(np.int32)
    assert offs[-1] <= M
    _per_group_case(M, K, offs, seed=M % 83)


def test_per_group_nan_column():
    x = torch.randn(64, 16).to(torch.bfloat16)
    xb = bits_of(x).copy()
    xb[10, 3] = 0x7FC0
    xt = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16)
    q, s = gpu_per_group(xt, [32, 64], mxq.ROW_MAJOR)
    qr, sr = oracle.per_group_quant(xb, [32, 64], mxq.ROW_MAJOR)
    assert np.isnan(s[0, 3]) and np.isnan(sr[0, 3])
    keep = np.ones(16, bool)
    keep[3] = False
    assert same_f32(s[:, keep], sr[:, keep]) and same_f32(s[1], sr[1])
    np.testing.assert_array_equal(q[:, keep], qr[:, keep])
    np.testing.assert_array_equal(q[32:], qr[32:])


# ---- the convert instruction itself -----------------------------------------------------------

def test_e4m3_convert_exhaustive_critical_range():
    """Every fp32 bit pattern with magnitude in [2^-11, 512] (both signs), plus a
    strided sample of all other finite patterns: the hardware convert the kernels use
    against the oracle encoder (ties, sign of zero, saturation)."""
    def run(bits_np):
        xd = torch.from_numpy(bits_np.view(np.int32)).cuda().view(torch.float32)
        qd = torch.empty(bits_np.size, dtype=torch.uint8, device="cuda")
        mxq.mx_e4m3_encode_f32(xd, qd)
        torch.cuda.synchronize()
        return qd.cpu().numpy()
    lo, hi = 0x3A000000, 0x44000001
    step = 1 << 24
    for start in range(lo, hi, step):
        b = np.arange(start, min(start + step, hi), dtype=np.uint32)
        for sgn in (0, 0x80000000):
            bb = b | np.uint32(sgn)
            np.testing.assert_array_equal(run(bb), oracle.e4m3_encode_f32(bb.view(np.float32)))
    rest = np.arange(0, 2 ** 32, 997, dtype=np.uint64).astype(np.uint32)
    f = rest.view(np.float32)
    rest = rest[np.isfinite(f)]
    np.testing.assert_array_equal(run(rest), oracle.e4m3_encode_f32(rest.view(np.float32)))
    nan = np.array([0x7FC00000, 0xFFC00000, 0x7F800001], dtype=np.uint32)
    assert np.all((run(nan) & 0x7F) == 0x7F)


def test_zero_size_calls_are_no_ops():
    x = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    e = torch.empty(0, dtype=torch.uint8, device="cuda")
    mxq.mx_quantize(x, 3, q_row=e, s_row=e, q_col=e, s_col=e)
    mxq.mx_dequantize(e, e, 1, 0, 64, 1, torch.empty(0, dtype=torch.bfloat16, device="cuda"))
    # M = 0 with groups: every group is empty, scales are still written
    s = torch.full((3, 16), float("nan"), device="cuda")
    mxq.fp8_per_group_rowwise_quant(torch.empty(0, 16, dtype=torch.bfloat16, device="cuda"),
                                    torch.tensor([0, 0, 5], dtype=torch.int32, device="cuda"),
                                    mxq.ROW_MAJOR, e, s)
    torch.cuda.synchronize()
    assert torch.all(s == torch.tensor(448.0) / torch.tensor(1e-12, dtype=torch.float32)).item()


def test_runs_on_a_side_stream():
    x = mixed(1, 256, 256, seed=21)
    st = torch.cuda.Stream()
    xd = x.cuda()
    out = mxq.empty_mx_outputs(xd, mxq.ROW)
    torch.cuda.synchronize()
    with torch.cuda.stream(st):
        mxq.mx_quantize(xd, mxq.ROW, **out)
    st.synchronize()
    ref = oracle.mx_quantize(bits_of(x), mxq.ROW)
    np.testing.assert_array_equal(out["q_row"].cpu().numpy()[0], ref["q_row"])


def test_zz_no_bounded_wait_gave_up():
    """Every tile copy of the tests above completed within its bounded wait."""
    assert mxq.mxq_wait_timeouts() == 0


@pytest.mark.parametrize("rows", [1, 31, 100, 1027])
def test_row_blocks_any_number_of_rows(rows):
    """1x32 blocks alone take any number of rows (an all-to-all split's token count)."""
    x = mixed(1, 32 * ((rows + 31) // 32), 160, seed=rows)[:rows].contiguous()
    xb = bits_of(x)
    got = gpu_mx_quantize(x, mxq.ROW)
    ref = oracle.mx_quantize(xb, oracle.ROW)
    assert_mx_equal(got, ref, ("q_row", "s_row"))
    y = gpu_mx_dequantize(ref["q_row"], ref["s_row"], 1, rows, 160, mxq.ROW)
    np.testing.assert_array_equal(y, oracle.mx_dequantize(ref["q_row"], ref["s_row"], 1, rows, 160, oracle.ROW))
