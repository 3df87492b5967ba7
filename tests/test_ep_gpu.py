"""The MXFP8 all-to-all on one GPU with the library's CUDA codec over NCCL.

With a world of one rank the exchange sends every token to itself, so the result must
be exactly the oracle's 1x32 quantize/dequantize of each token, forward and backward;
this checks the CUDA codec, the byte tensors through NCCL and the split plumbing on
real hardware.  (More ranks need more GPUs; the routing itself is covered on CPU
process groups.)
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle

from _gpu import bits_of, ensure_lib

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module")
def nccl_group():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ensure_lib()
    import datetime
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    yield
    dist.destroy_process_group()


def _oracle_round_trip(x_bits: np.ndarray) -> np.ndarray:
    r = oracle.mx_quantize(x_bits, oracle.ROW)
    T, D = x_bits.shape
    return oracle.mx_dequantize(r["q_row"], r["s_row"], 1, T, D, oracle.ROW).reshape(T, D)


@pytest.mark.parametrize("T,D", [(0, 32), (1, 32), (37, 160), (4099, 5120)])
def test_all_to_all_one_rank(nccl_group, T, D):
    from mxfp8_quantization_moe_mx_b200 import ep
    g = torch.Generator().manual_seed(T + D)
    x = (torch.randn(T, D, generator=g) * torch.exp(torch.randn(T, 1, generator=g))).to(torch.bfloat16)
    gy = torch.randn(T, D, generator=g).to(torch.bfloat16)
    in_splits, out_splits = ep.exchange_splits(torch.tensor([T], dtype=torch.int64, device="cuda"))
    assert in_splits == [T] and out_splits == [T]
    xd = x.cuda().requires_grad_(True)
    y = ep.mxfp8_all_to_all(xd, out_splits, in_splits)
    y.backward(gy.cuda())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bits_of(y.detach()), _oracle_round_trip(bits_of(x)))
    np.testing.assert_array_equal(bits_of(xd.grad), _oracle_round_trip(bits_of(gy)))


def test_all_gather_one_rank(nccl_group):
    from mxfp8_quantization_moe_mx_b200 import ep
    g = torch.Generator().manual_seed(3)
    x = torch.randn(100, 320, generator=g).to(torch.bfloat16)
    xd = x.cuda().requires_grad_(True)
    y = ep.mxfp8_all_gather(xd)
    y.backward(torch.ones_like(y))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bits_of(y.detach()), _oracle_round_trip(bits_of(x)))
    assert torch.all(xd.grad == 1).item()
