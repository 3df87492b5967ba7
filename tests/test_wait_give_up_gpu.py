"""The per-group kernels' bounded waits, made to give up on purpose.

With the wait limit set to 0 every bounded wait (a CTA's wait for the TMA copy of its
tile, and in a thread-block cluster the wait for the siblings' partial maxima) gives
up at once.  The CTA then waits, with its own long limit, for the copies still in
flight, and skips its (group, column-slab) tile; in a cluster the whole cluster skips
it.  This file checks the contract that follows on each kernel shape:

  * no code byte of a skipped tile is written and no scale of it is written, so a
    caller that pre-fills the outputs sees only the fill there (never codes derived
    from incomplete maxima);
  * tiles that needed no wait (a CTA whose groups are all empty) are still exact;
  * the give-up count grows by exactly the number of CTAs that gave up, and no copy
    was abandoned;
  * with the default limit back, the same call is bit-exact again and counts nothing.

No GPU fault is involved: giving up is an ordinary branch of the kernels, and every
copy still lands before its CTA exits.
"""
import numpy as np
import pytest
import torch

import oracle
import mxfp8_quantization_moe_mx_b200 as mxq
from mxfp8_quantization_moe_mx_b200 import workloads as wl

from _gpu import CANARY, bits_of, ensure_lib, gpu_per_group, same_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ensure_lib()
    yield
    mxq.mxq_set_wait_limit_ns(mxq.WAIT_LIMIT_DEFAULT_NS)


def _expected_give_ups(plan, K, start, end):
    """CTAs that give up when every wait gives up at once: a CTA waits for its tile
    only if its rows are not empty; in a cluster every CTA also waits for the
    siblings' maxima."""
    slabs = (K + plan["slab_cols"] - 1) // plan["slab_cols"]
    sizes = end - start
    if plan["kernel"] == "pair":
        pairs = [sizes[i:i + 2].sum() for i in range(0, len(sizes), 2)]
        return slabs * sum(1 for p in pairs if p > 0)
    if plan["cluster"] > 1:
        return slabs * plan["cluster"] * len(sizes)
    return slabs * int(np.count_nonzero(sizes))


@pytest.mark.parametrize("M,K,sizes,layout,kernel,cluster", [
    # one CTA per (group, 64-column slab), row-major; an empty group needs no wait
    (1024, 256, [250, 0, 260, 255, 259], mxq.ROW_MAJOR, "tile", 1),
    # 1024-row groups: tiles split over a cluster of four CTAs
    (4096, 192, [1000, 1100, 0, 996, 1000], mxq.ROW_MAJOR, "tile", 4),
    # column-major, ~128-row groups: two groups per CTA; the last pair is empty
    (1024, 256, [120, 130, 0, 140, 126, 128, 120, 130, 0, 0], mxq.COL_MAJOR, "pair", 1),
])
def test_give_up_skips_whole_tiles(M, K, sizes, layout, kernel, cluster):
    offs = np.cumsum(np.asarray(sizes)).astype(np.int32)
    G = len(sizes)
    plan = mxq.fp8_per_group_rowwise_plan(M, K, G, layout)
    assert plan["kernel"] == kernel and plan["cluster"] == cluster, plan
    x = wl.stress(seed=M + K, M=M, K=K, n_groups=3, n_empty=0)["x"]
    xb = bits_of(x)
    start, end = oracle.group_bounds(offs, M)
    shape = (M, K) if layout == mxq.ROW_MAJOR else (K, M)
    qr, sr = oracle.per_group_quant(xb, offs, layout, q_init=np.full(shape, CANARY))

    before, lost_before = mxq.mxq_wait_timeouts(), mxq.mxq_wait_abandoned()
    mxq.mxq_set_wait_limit_ns(0)
    try:
        q, s = gpu_per_group(x, offs, layout)
    finally:
        mxq.mxq_set_wait_limit_ns(mxq.WAIT_LIMIT_DEFAULT_NS)
    gave_up = mxq.mxq_wait_timeouts() - before
    assert gave_up == _expected_give_ups(plan, K, start, end)
    assert mxq.mxq_wait_abandoned() == lost_before

    # every CTA with rows gave up: no code byte anywhere was written
    assert np.all(q == CANARY)
    # a group's scales are untouched (NaN fill) when its CTA gave up, exact otherwise
    for g in range(G):
        if np.all(np.isnan(s[g])):
            continue
        assert end[g] == start[g] and plan["cluster"] == 1, f"group {g} wrote scales after giving up"
        if plan["kernel"] == "pair":
            mate = g ^ 1
            assert mate >= G or end[mate] == start[mate]
        assert same_f32(s[g], sr[g]), g

    # the default limit again: bit-exact, nothing counted
    before = mxq.mxq_wait_timeouts()
    q, s = gpu_per_group(x, offs, layout)
    assert same_f32(s, sr)
    np.testing.assert_array_equal(q, qr)
    assert mxq.mxq_wait_timeouts() == before
