"""GPU parity of the layout calls between the quantizers and the scaled grouped GEMM:
the byte transpose (column-major per-group codes -> row-major) and the 128 x 4 tiled
E8M0 scale layout of the block-scaled MMA.  Both are byte moves, so the comparison
with the oracle is exact; output buffers are canary-filled and their guard bytes
checked."""
import numpy as np
import pytest
import torch

import oracle
import mxfp8_quantization_moe_mx_b200 as mxq
from mxfp8_quantization_moe_mx_b200 import workloads as wl

from _gpu import CANARY, bits_of, ensure_lib

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ensure_lib()


def gpu_transpose(x: np.ndarray, src_offset: int = 0, dst_offset: int = 0, guard: int = 64) -> np.ndarray:
    """x (batch, rows, cols) uint8 through mxq_transpose_u8, with the source and the
    destination placed `*_offset` bytes into their buffers (alignment cases)."""
    b, r, c = x.shape
    n = x.size
    sb = torch.zeros(n + src_offset, dtype=torch.uint8, device="cuda")
    sb[src_offset:] = torch.from_numpy(x.reshape(-1)).cuda()
    db = torch.full((n + dst_offset + 2 * guard,), CANARY, dtype=torch.uint8, device="cuda")
    src = sb[src_offset:].view(b, r, c)
    dst = db[guard + dst_offset:guard + dst_offset + n]
    mxq.mxq_transpose_u8(src, dst)
    torch.cuda.synchronize()
    h = db.cpu().numpy()
    assert np.all(h[:guard + dst_offset] == CANARY) and np.all(h[guard + dst_offset + n:] == CANARY)
    return h[guard + dst_offset:guard + dst_offset + n].reshape(b, c, r)


@pytest.mark.parametrize("shape", [(1, 16, 16), (1, 256, 128), (2, 48, 80), (1, 512, 400), (3, 272, 144),
                                   (1, 33, 17), (2, 1001, 136), (1, 7, 1), (1, 1, 300)])
def test_transpose_shapes(shape):
    x = np.random.default_rng(sum(shape)).integers(0, 256, shape, dtype=np.uint8)
    np.testing.assert_array_equal(gpu_transpose(x), oracle.transpose_u8(x))


@pytest.mark.parametrize("src_offset,dst_offset", [(1, 0), (0, 8), (4, 4)])
def test_transpose_misaligned_pointers(src_offset, dst_offset):
    x = np.random.default_rng(3).integers(0, 256, (2, 64, 48), dtype=np.uint8)
    np.testing.assert_array_equal(gpu_transpose(x, src_offset, dst_offset), oracle.transpose_u8(x))


def test_column_major_per_group_then_transpose_is_row_major():
    """The pages' route for many groups: column-major per-group codes, then the
    transform, give the oracle's row-major codes (groups cover every row)."""
    g = torch.Generator().manual_seed(5)
    M, K, G = 3000, 320, 24
    offs = wl.uniform_group_offsets(g, M, G).numpy()
    x = wl.per_group(seed=77, M=M, K=K, n_groups=G)["x"]
    xd = x.cuda()
    q = torch.empty(K, M, dtype=torch.uint8, device="cuda")
    s = torch.empty(G, K, dtype=torch.float32, device="cuda")
    mxq.fp8_per_group_rowwise_quant(xd, torch.from_numpy(offs).cuda(), mxq.COL_MAJOR, q, s)
    qt = torch.empty(M, K, dtype=torch.uint8, device="cuda")
    mxq.mxq_transpose_u8(q, qt)
    torch.cuda.synchronize()
    qr, _ = oracle.per_group_quant(bits_of(x), offs, oracle.ROW_MAJOR)
    np.testing.assert_array_equal(qt.cpu().numpy(), qr)


def gpu_blocked(s: np.ndarray, offs=None, guard: int = 64) -> np.ndarray:
    b, r, k = s.shape
    G = 0 if offs is None else len(offs)
    n = mxq.mx_scales_blocked_bytes(b, r, k, G)
    assert n == oracle.mx_scales_blocked_bytes(b, r, k, G)
    ob = torch.full((n + 2 * guard,), 0xEE, dtype=torch.uint8, device="cuda")
    od = None if offs is None else torch.as_tensor(np.asarray(offs, np.int32)).cuda()
    mxq.mx_scales_to_blocked(torch.from_numpy(s).cuda(), ob[guard:guard + n], od)
    torch.cuda.synchronize()
    h = ob.cpu().numpy()
    assert np.all(h[:guard] == 0xEE) and np.all(h[guard + n:] == 0xEE)
    return h[guard:guard + n]


@pytest.mark.parametrize("shape", [(1, 128, 4), (1, 130, 5), (3, 200, 6), (2, 1024, 160), (1, 1, 1),
                                   (16, 256, 160)])
def test_blocked_scales_per_matrix(shape):
    s = np.random.default_rng(sum(shape)).integers(0, 256, shape, dtype=np.uint8)
    np.testing.assert_array_equal(gpu_blocked(s), oracle.mx_scales_to_blocked(s, fill=0xEE))


@pytest.mark.parametrize("rows,nk,offs", [
    (700, 10, [100, 100, 356, 700]),            # empty group, exact cover
    (700, 12, [0, 129, 600]),                   # leading empty group, trailing rows
    (700, 7, [650, 640, 900, -3]),              # malformed: decreasing, past the end, negative
    (4096, 160, list(range(32, 4097, 32))),     # 128 groups of 32 rows: every group its own tile
    (5000, 160, [1, 2, 3, 4, 4, 4, 5000]),
])
def test_blocked_scales_per_group(rows, nk, offs):
    s = np.random.default_rng(rows + nk).integers(0, 256, (1, rows, nk), dtype=np.uint8)
    np.testing.assert_array_equal(gpu_blocked(s, offs), oracle.mx_scales_to_blocked(s, offs, fill=0xEE))


def test_blocked_scales_at_the_dispatch_payload_size():
    """Scales of the (65536, 5120) dispatch payload's shape (65536 x 160 bytes, seeded
    random bytes), laid out per expert with the payload's 16 expert offsets."""
    offs = wl.dispatch(rows=65536, cols=32)["offs"].numpy()
    s = np.random.default_rng(8).integers(0, 256, (1, 65536, 160), dtype=np.uint8)
    np.testing.assert_array_equal(gpu_blocked(s, offs), oracle.mx_scales_to_blocked(s, offs, fill=0xEE))
