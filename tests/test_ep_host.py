"""The MXFP8 expert-parallel all-to-all on CPU process groups (gloo, world size 2).

The product codec is the CUDA kernels; here each rank passes a codec built on the
oracle (test infrastructure), so what is checked is the exchange itself: the split
bookkeeping (the counts' all-to-all and the device-to-host lists), that codes and
scales travel with the same splits, that every token lands where the reference
routing puts it -- bit-exactly equal to the oracle's quantize/dequantize of that
token -- and that the backward pass sends the gradient back through the reverse
exchange.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle


class OracleCodec:
    """1x32 MX quantize / dequantize by the CPU oracle (CPU tensors)."""

    def quantize(self, x):
        bits = x.contiguous().view(torch.int16).numpy().view(np.uint16)
        r = oracle.mx_quantize(bits, oracle.ROW)
        return torch.from_numpy(r["q_row"].copy()), torch.from_numpy(r["s_row"].copy())

    def dequantize(self, q, s):
        T, D = q.shape
        y = oracle.mx_dequantize(q.numpy(), s.numpy(), 1, T, D, oracle.ROW)
        return torch.from_numpy(y.reshape(T, D).view(np.int16).copy()).view(torch.bfloat16)


def _round_trip(x: torch.Tensor) -> np.ndarray:
    c = OracleCodec()
    return c.dequantize(*c.quantize(x)).view(torch.int16).numpy().view(np.uint16)


def _inputs(rank, D):
    g = torch.Generator().manual_seed(100 + rank)
    T = [37, 50][rank]
    x = (torch.randn(T, D, generator=g) * torch.exp(torch.randn(T, 1, generator=g))).to(torch.bfloat16)
    counts = [[20, 17], [0, 50]][rank]      # rank 1 sends nothing to rank 0
    gy = torch.randn(sum([[20, 0], [17, 50]][rank]), D, generator=g).to(torch.bfloat16)
    return x, counts, gy


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from mxfp8_quantization_moe_mx_b200 import ep
        D = 96
        x, counts, gy = _inputs(rank, D)
        in_splits, out_splits = ep.exchange_splits(torch.tensor(counts, dtype=torch.int64))
        xr = x.clone().requires_grad_(True)
        y = ep.mxfp8_all_to_all(xr, out_splits, in_splits, codec=OracleCodec())
        y.backward(gy)
        # the MXFP8 all-gather of each rank's first 24 tokens, and its bf16 backward
        xg = x[:24].clone().requires_grad_(True)
        yg = ep.mxfp8_all_gather(xg, codec=OracleCodec())
        gg = torch.full(yg.shape, 0.5 + rank, dtype=torch.bfloat16)
        yg.backward(gg)
        q.put((rank, in_splits, out_splits, y.detach().view(torch.int16).numpy().copy(),
               xr.grad.view(torch.int16).numpy().copy(), yg.detach().view(torch.int16).numpy().copy(),
               xg.grad.float().numpy().copy()))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module")
def results():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(world):
        r = q.get(timeout=180)
        out[r[0]] = r[1:]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return out


def test_split_exchange(results):
    assert results[0][0] == [20, 17] and results[0][1] == [20, 0]
    assert results[1][0] == [0, 50] and results[1][1] == [17, 50]


def test_tokens_land_quantized_where_routed(results):
    D = 96
    xs = [_inputs(r, D)[0] for r in range(2)]
    # rank 0 receives rank 0's first 20 tokens; rank 1 receives rank 0's last 17 then rank 1's 50
    expect = {0: xs[0][:20], 1: torch.cat([xs[0][20:], xs[1]])}
    for r in range(2):
        got = results[r][2].view(np.uint16)
        np.testing.assert_array_equal(got, _round_trip(expect[r]))


def test_gradient_goes_back_through_the_reverse_exchange(results):
    D = 96
    gys = [_inputs(r, D)[2] for r in range(2)]
    # rank 0's tokens: first 20 went to rank 0 (rows 0..19 of its output), the last 17
    # to rank 1 (rows 0..16 there); rank 1's 50 tokens went to rank 1 (rows 17..66)
    expect = {0: torch.cat([gys[0][:20], gys[1][:17]]), 1: gys[1][17:]}
    for r in range(2):
        got = results[r][3].view(np.uint16)
        np.testing.assert_array_equal(got, _round_trip(expect[r]))


def test_wire_bytes():
    from mxfp8_quantization_moe_mx_b200 import ep
    b = ep.wire_bytes(8 * 8192, 5120)
    assert b["bf16"] == 2 * 65536 * 5120 and b["mxfp8"] == 65536 * 5120 * 33 // 32


def test_all_gather_in_mxfp8(results):
    D = 96
    shards = [_inputs(r, D)[0][:24] for r in range(2)]
    expect = _round_trip(torch.cat(shards))
    for r in range(2):
        np.testing.assert_array_equal(results[r][4].view(np.uint16), expect)


def test_all_gather_backward_is_a_bf16_reduce_scatter(results):
    # each rank's output gradient is 0.5 + rank everywhere: the summed shard gradient is 2.0
    for r in range(2):
        assert np.all(results[r][5] == 2.0)
