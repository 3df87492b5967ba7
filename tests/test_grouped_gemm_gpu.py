"""GPU parity of the MXFP8 grouped GEMM (tcgen05 block-scaled MMA) against the oracle.

Inputs are seeded bf16 tokens and expert weights, quantized to MXFP8 and laid out by
the oracle (for the oracle-input tests) or by the CUDA path itself (for the chained
test, compared with the oracle's own chain).  The oracle sums the exact products in
double; the tensor cores accumulate in fp32 and the result is rounded once to bf16,
so each output must satisfy

    |gpu - ref| <= 2^-8 |ref| + K * 2^-23 * sum_k |a_k b_k|

(2^-9 |ref| is the bf16 rounding, K * 2^-24 * sum |a_k b_k| bounds any order of fp32
additions; both doubled for slack).  Rows in no group must keep their canary value.
"""
import numpy as np
import pytest
import torch

import oracle
import mxfp8_quantization_moe_mx_b200 as mxq
from mxfp8_quantization_moe_mx_b200 import workloads as wl

from _gpu import bits_of, ensure_lib

pytestmark = pytest.mark.gpu

CANARY_BF16 = 0x7FBF  # a NaN pattern the kernel never writes


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ensure_lib()
    before = mxq.mxq_wait_timeouts()
    yield
    assert mxq.mxq_wait_timeouts() == before


def _bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    with np.errstate(invalid="ignore"):
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _operands(M, N, K, G, seed):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(M, K, generator=g) * torch.exp(torch.randn(M, 1, generator=g))).to(torch.bfloat16)
    w = (torch.randn(G, N, K, generator=g) * 0.02).to(torch.bfloat16)
    return x, w


def _run_gpu(qa, sfa_blk, qb, sfb_blk, offs, M, N):
    out = torch.full((M, N), CANARY_BF16, dtype=torch.int16, device="cuda")
    o = out.view(torch.bfloat16)
    mxq.mx_grouped_gemm(torch.from_numpy(qa).cuda(), torch.from_numpy(sfa_blk).cuda(),
                        torch.from_numpy(qb).cuda(), torch.from_numpy(sfb_blk).cuda(),
                        torch.as_tensor(np.asarray(offs, np.int32)).cuda(), o)
    torch.cuda.synchronize()
    return out.cpu().numpy().view(np.uint16)


def _check(got_bits, ref, mag, K, rows_in_groups):
    got = _bf16_to_f64(got_bits)
    tol = 2.0 ** -8 * np.abs(ref) + K * 2.0 ** -23 * mag
    inside = np.zeros(got.shape[0], bool)
    inside[rows_in_groups] = True
    err = np.abs(got[inside] - ref[inside])
    bad = err > tol[inside]
    assert not bad.any(), f"{bad.sum()} outputs out of tolerance; worst excess {np.max(err - tol[inside]):.3g}"
    assert np.all(got_bits[~inside] == CANARY_BF16), "rows in no group were written"


@pytest.mark.parametrize("M,N,K,sizes", [
    (128, 256, 128, [128]),                          # one tile
    (320, 256, 256, [100, 0, 150]),                  # empty group, partial tiles, trailing rows
    (1024, 512, 640, [129, 1, 257, 383, 230]),       # ragged groups, two N tiles, five K blocks
    (704, 256, 1024, [650, 40]),                     # a group larger than five tiles
])
def test_grouped_gemm_against_oracle(M, N, K, sizes):
    G = len(sizes)
    offs = np.cumsum(sizes).astype(np.int32)
    x, w = _operands(M, N, K, G, seed=M + N + K)
    ra = oracle.mx_quantize(bits_of(x), oracle.ROW)
    rb = oracle.mx_quantize(bits_of(w), oracle.ROW)
    sfa_blk = oracle.mx_scales_to_blocked(ra["s_row"], offs)
    sfb_blk = oracle.mx_scales_to_blocked(rb["s_row"])
    got = _run_gpu(ra["q_row"], sfa_blk, rb["q_row"], sfb_blk, offs, M, N)
    ref, mag = oracle.mx_grouped_gemm(ra["q_row"], ra["s_row"], rb["q_row"], rb["s_row"], offs)
    start, end = oracle.group_bounds(offs, M)
    rows = np.concatenate([np.arange(a, b) for a, b in zip(start, end)])
    _check(got, ref, mag, K, rows)


def test_grouped_gemm_several_units_per_cluster():
    """More 256 x 256 units than CTA pairs, so pairs walk two units (the accumulator
    handed from one unit's epilogue to the next unit's MMAs), and more than 32 groups
    (the unit lookup scans the offsets 32 at a time): 40 groups with odd and even tile
    counts, empty groups among them, compared whole."""
    rng = np.random.default_rng(40)
    sizes = rng.integers(0, 260, size=40)
    sizes[[3, 17, 18, 39]] = 0
    sizes[5] = 128 * 3 + 1          # four tiles, the last with one row
    M, N, K = int(sizes.sum()) + 50, 768, 128
    offs = np.cumsum(sizes).astype(np.int32)
    pairs = sum(((int(n) + 127) // 128 + 1) // 2 for n in sizes)
    assert pairs * (N // 256) > torch.cuda.get_device_properties(0).multi_processor_count // 2
    x, w = _operands(M, N, K, len(sizes), seed=41)
    ra = oracle.mx_quantize(bits_of(x), oracle.ROW)
    rb = oracle.mx_quantize(bits_of(w), oracle.ROW)
    got = _run_gpu(ra["q_row"], oracle.mx_scales_to_blocked(ra["s_row"], offs), rb["q_row"],
                   oracle.mx_scales_to_blocked(rb["s_row"]), offs, M, N)
    ref, mag = oracle.mx_grouped_gemm(ra["q_row"], ra["s_row"], rb["q_row"], rb["s_row"], offs)
    start, end = oracle.group_bounds(offs, M)
    rows = np.concatenate([np.arange(a, b) for a, b in zip(start, end)])
    _check(got, ref, mag, K, rows)


def test_grouped_gemm_no_rows_in_any_group():
    """Every group empty: no unit at all, the output keeps its canary."""
    M, N, K = 256, 256, 128
    offs = np.zeros(3, np.int32)
    x, w = _operands(M, N, K, 3, seed=9)
    ra = oracle.mx_quantize(bits_of(x), oracle.ROW)
    rb = oracle.mx_quantize(bits_of(w), oracle.ROW)
    sfa = np.zeros(mxq.mx_scales_blocked_bytes(1, M, K // 32, 3), np.uint8)
    got = _run_gpu(ra["q_row"], sfa, rb["q_row"], oracle.mx_scales_to_blocked(rb["s_row"]), offs, M, N)
    assert np.all(got == CANARY_BF16)


def test_grouped_gemm_one_group_odd_tiles():
    """One group of three M tiles (the second CTA of the last pair multiplies filler and
    stores nothing) followed by rows in no group."""
    M, N, K = 420, 512, 256
    offs = np.array([300], np.int32)
    x, w = _operands(M, N, K, 1, seed=13)
    ra = oracle.mx_quantize(bits_of(x), oracle.ROW)
    rb = oracle.mx_quantize(bits_of(w), oracle.ROW)
    got = _run_gpu(ra["q_row"], oracle.mx_scales_to_blocked(ra["s_row"], offs), rb["q_row"],
                   oracle.mx_scales_to_blocked(rb["s_row"]), offs, M, N)
    ref, mag = oracle.mx_grouped_gemm(ra["q_row"], ra["s_row"], rb["q_row"], rb["s_row"], offs)
    _check(got, ref, mag, K, np.arange(300))


def test_grouped_gemm_malformed_offsets():
    """Decreasing, negative and past-the-end offsets follow the clamp rule."""
    M, N, K = 416, 256, 256
    offs = np.array([120, 60, -4, 390, 900], np.int32)
    G = offs.size
    x, w = _operands(M, N, K, G, seed=5)
    ra = oracle.mx_quantize(bits_of(x), oracle.ROW)
    rb = oracle.mx_quantize(bits_of(w), oracle.ROW)
    got = _run_gpu(ra["q_row"], oracle.mx_scales_to_blocked(ra["s_row"], offs), rb["q_row"],
                   oracle.mx_scales_to_blocked(rb["s_row"]), offs, M, N)
    ref, mag = oracle.mx_grouped_gemm(ra["q_row"], ra["s_row"], rb["q_row"], rb["s_row"], offs)
    start, end = oracle.group_bounds(offs, M)
    rows = np.concatenate([np.arange(a, b) for a, b in zip(start, end)])
    _check(got, ref, mag, K, rows)


def test_grouped_gemm_chain_on_the_gpu():
    """Tokens and weights quantized, and their scales laid out, by the CUDA path; the
    oracle runs the same chain from the same bf16 inputs."""
    M, N, K, G = 1024, 256, 512, 8
    gen = torch.Generator().manual_seed(17)
    offs = wl.uniform_group_offsets(gen, M, G)
    x, w = _operands(M, N, K, G, seed=17)
    xd, wd, od = x.cuda(), w.cuda(), offs.cuda()
    oa = mxq.empty_mx_outputs(xd, mxq.ROW)
    ob = mxq.empty_mx_outputs(wd, mxq.ROW)
    mxq.mx_quantize(xd, mxq.ROW, **oa)
    mxq.mx_quantize(wd, mxq.ROW, **ob)
    sfa = torch.empty(mxq.mx_scales_blocked_bytes(1, M, K // 32, G), dtype=torch.uint8, device="cuda")
    sfb = torch.empty(mxq.mx_scales_blocked_bytes(G, N, K // 32, 0), dtype=torch.uint8, device="cuda")
    mxq.mx_scales_to_blocked(oa["s_row"][0], sfa, od)
    mxq.mx_scales_to_blocked(ob["s_row"], sfb)
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    mxq.mx_grouped_gemm(oa["q_row"][0], sfa, ob["q_row"], sfb, od, out)
    torch.cuda.synchronize()
    ra = oracle.mx_quantize(bits_of(x), oracle.ROW)
    rb = oracle.mx_quantize(bits_of(w), oracle.ROW)
    ref, mag = oracle.mx_grouped_gemm(ra["q_row"], ra["s_row"], rb["q_row"], rb["s_row"], offs.numpy())
    _check(bits_of(out), ref, mag, K, np.arange(M))


@pytest.mark.slow
def test_grouped_gemm_at_the_llama4_expert_shape():
    """The launch the benchmark times: dispatch-payload tokens (65536, 5120) over 16
    groups x 16 expert matrices (8192, 5120), every operand quantized and laid out by
    the CUDA path.  The oracle recomputes 64 sampled rows (4 per group) x 256 sampled
    columns from the seeded bf16 inputs (MX row blocks and output entries are
    independent of the rows and columns left out)."""
    M, K, N, G = 65536, 5120, 8192, 16
    t = wl.dispatch(rows=M, cols=K, n_groups=G)
    x, offs = t["x"], t["offs"].numpy()
    w = wl.dual_axis(act_rows=32, dim=K, experts=G, hidden=N)["w"]
    xd, wd, od = x.cuda(), w.cuda(), torch.from_numpy(offs).cuda()
    oa = mxq.empty_mx_outputs(xd, mxq.ROW)
    ob = mxq.empty_mx_outputs(wd, mxq.ROW)
    mxq.mx_quantize(xd, mxq.ROW, **oa)
    mxq.mx_quantize(wd, mxq.ROW, **ob)
    sfa = torch.empty(mxq.mx_scales_blocked_bytes(1, M, K // 32, G), dtype=torch.uint8, device="cuda")
    sfb = torch.empty(mxq.mx_scales_blocked_bytes(G, N, K // 32, 0), dtype=torch.uint8, device="cuda")
    mxq.mx_scales_to_blocked(oa["s_row"][0], sfa, od)
    mxq.mx_scales_to_blocked(ob["s_row"], sfb)
    del xd, wd
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    mxq.mx_grouped_gemm(oa["q_row"][0], sfa, ob["q_row"], sfb, od, out)
    torch.cuda.synchronize()

    rng = np.random.default_rng(31)
    start, end = oracle.group_bounds(offs, M)
    rows = np.concatenate([np.sort(rng.choice(np.arange(a, b), 4, replace=False)) for a, b in zip(start, end)])
    # the first and last row of the first group, the last row of the last group
    rows[0], rows[1], rows[-1] = start[0], end[0] - 1, end[-1] - 1
    cols = np.sort(rng.choice(N, 256, replace=False))
    cols[-1] = N - 1
    ra = oracle.mx_quantize(np.ascontiguousarray(bits_of(x)[rows]), oracle.ROW)
    rb = oracle.mx_quantize(np.ascontiguousarray(bits_of(w)[:, cols, :]), oracle.ROW)
    sub_offs = np.cumsum([4] * G).astype(np.int32)
    ref, mag = oracle.mx_grouped_gemm(ra["q_row"], ra["s_row"], rb["q_row"], rb["s_row"], sub_offs)
    idx_r = torch.as_tensor(rows, device="cuda")
    idx_c = torch.as_tensor(cols, device="cuda")
    got = bits_of(out.index_select(0, idx_r).index_select(1, idx_c))
    _check(got, ref, mag, K, np.arange(len(rows)))
