"""GPU parity of fp8_per_group_rowwise_quant_batched: a 3-D tensor of E matrices, each
matrix its own group, row-major (E, M, K) or per-matrix column-major (E, K, M) codes,
bit for bit against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import mxfp8_quantization_moe_mx_b200 as mxq
from mxfp8_quantization_moe_mx_b200 import workloads as wl

from _gpu import CANARY, bits_of, ensure_lib, same_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ensure_lib()


def _run(x, layout, guard=64):
    E, M, K = x.shape
    n = E * M * K
    qb = torch.full((n + 2 * guard,), CANARY, dtype=torch.uint8, device="cuda")
    sb = torch.full((E * K + 2 * guard,), float("nan"), dtype=torch.float32, device="cuda")
    mxq.fp8_per_group_rowwise_quant_batched(x.cuda(), layout, qb[guard:guard + n], sb[guard:guard + E * K])
    torch.cuda.synchronize()
    qh, sh = qb.cpu().numpy(), sb.cpu().numpy()
    assert np.all(qh[:guard] == CANARY) and np.all(qh[-guard:] == CANARY)
    assert np.all(np.isnan(sh[:guard])) and np.all(np.isnan(sh[-guard:]))
    shape = (E, M, K) if layout == mxq.ROW_MAJOR else (E, K, M)
    return qh[guard:-guard].reshape(shape), sh[guard:-guard].reshape(E, K)


@pytest.mark.parametrize("E,M,K", [(1, 64, 64), (3, 100, 72), (4, 1001, 136), (16, 256, 320), (2, 5000, 64),
                                   (5, 37, 8), (8, 4096, 128)])
def test_batched_per_group(E, M, K):
    x = wl.stress(seed=E * M + K, M=E * M, K=K if K % 32 == 0 else K + 32 - K % 32, n_groups=3,
                  n_empty=0)["x"][:, :K].contiguous().view(E, M, K)
    xb = bits_of(x).reshape(E, M, K)
    for layout in (mxq.ROW_MAJOR, mxq.COL_MAJOR):
        q, s = _run(x, layout)
        qr, sr = oracle.per_group_quant_batched(xb, layout)
        assert same_f32(s, sr), (E, M, K, layout)
        np.testing.assert_array_equal(q, qr, err_msg=f"E={E} M={M} K={K} layout={layout}")


def test_batched_expert_weights_shape():
    """The expert weights of the Llama4 debug model, (16, 8192, 5120), column-major."""
    w = wl.dual_axis()["w"]
    E, M, K = w.shape
    q, s = _run(w, mxq.COL_MAJOR)
    wb = bits_of(w).reshape(E, M, K)
    for e in (0, 7, 15):
        qr, sr = oracle.per_group_quant_batched(wb[e:e + 1], mxq.COL_MAJOR)
        assert same_f32(s[e:e + 1], sr)
        np.testing.assert_array_equal(q[e:e + 1], qr)
