"""The MXFP8 all-to-all on four CPU process groups (gloo) with seeded, uneven splits,
zeros among them and one rank that has no tokens at all: every token lands where the plain routing puts it, bit-exactly equal
to the oracle's 1x32 quantize/dequantize of that token, and the backward pass returns
each gradient row to the token it came from.  The codec is the oracle (test
infrastructure); the product codec is the CUDA kernels."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from test_ep_host import OracleCodec, _round_trip

WORLD, D = 4, 64


def _counts(rank):
    if rank == WORLD - 1:
        return [0] * WORLD             # a rank with no tokens at all
    g = np.random.default_rng(7 + rank)
    c = g.integers(0, 9, size=WORLD)
    c[(rank + 1) % WORLD] = 0          # every other rank sends nothing to one peer
    return [int(v) for v in c]


def _tokens(rank):
    g = torch.Generator().manual_seed(300 + rank)
    T = sum(_counts(rank))
    return (torch.randn(T, D, generator=g) * torch.exp(torch.randn(T, 1, generator=g))).to(torch.bfloat16)


def _grads(rank):
    g = torch.Generator().manual_seed(500 + rank)
    R = sum(_counts(src)[rank] for src in range(WORLD))
    return torch.randn(R, D, generator=g).to(torch.bfloat16)


def _worker(rank, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        from mxfp8_quantization_moe_mx_b200 import ep
        in_splits, out_splits = ep.exchange_splits(torch.tensor(_counts(rank), dtype=torch.int64))
        x = _tokens(rank).requires_grad_(True)
        y = ep.mxfp8_all_to_all(x, out_splits, in_splits, codec=OracleCodec())
        y.backward(_grads(rank))
        q.put((rank, in_splits, out_splits, y.detach().view(torch.int16).numpy().copy(),
               x.grad.view(torch.int16).numpy().copy()))
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def results():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(WORLD):
        r = q.get(timeout=240)
        out[r[0]] = r[1:]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return out


def test_splits_are_each_others_transpose(results):
    for r in range(WORLD):
        assert results[r][0] == _counts(r)
        assert results[r][1] == [_counts(src)[r] for src in range(WORLD)]


def test_forward_routes_every_token(results):
    xs = [_tokens(r) for r in range(WORLD)]
    for dst in range(WORLD):
        parts = []
        for src in range(WORLD):
            c = _counts(src)
            a = sum(c[:dst])
            parts.append(xs[src][a:a + c[dst]])
        np.testing.assert_array_equal(results[dst][2].view(np.uint16), _round_trip(torch.cat(parts)))


def test_backward_returns_every_gradient_row(results):
    gs = [_grads(r) for r in range(WORLD)]
    for src in range(WORLD):
        c = _counts(src)
        parts = []
        for dst in range(WORLD):
            # rank dst's output rows from src start after the rows from ranks < src
            a = sum(_counts(s)[dst] for s in range(src))
            parts.append(gs[dst][a:a + c[dst]])
        np.testing.assert_array_equal(results[src][3].view(np.uint16), _round_trip(torch.cat(parts)))
