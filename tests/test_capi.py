"""The C ABI without a GPU: libmxq.so loads, exports every function include/mxq.h
declares, and rejects bad arguments on the host before touching CUDA.

Only argument checks that come before any CUDA call are exercised here (fake but
aligned non-null pointers are never dereferenced on those paths); zero-size calls
return MXQ_OK without launching.
"""
import ctypes
import os
import re

import pytest

import mxfp8_quantization_moe_mx_b200 as mxq
from mxfp8_quantization_moe_mx_b200 import build as mxq_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mxq.h")

OK, NULL, SHAPE, ALIGN, ARG = 0, 1, 2, 3, 4
P = 0x10000   # a fake 16-byte-aligned "device" address; never dereferenced below
P8 = 0x10008  # 8-byte but not 16-byte aligned


@pytest.fixture(scope="module")
def L():
    mxq_build.build()
    return mxq.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:int|const char\*|size_t|void)\s+\**\s*(\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("mx_quantize", "mx_dequantize", "fp8_per_group_rowwise_quant", "mx_e4m3_encode_f32",
              "mxq_status_string", "mxq_last_cuda_error", "mxq_wait_timeouts", "fp8_per_group_rowwise_plan"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    # and exports them with C linkage (plain names in the dynamic symbol table)
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", mxq.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    for name in declared_functions():
        assert name in exported, name


def test_status_strings(L):
    for s in range(7):
        assert L.mxq_status_string(s).startswith(b"MXQ_")
    assert L.mxq_status_string(99) == b"unknown mxq status"


def test_mx_quantize_argument_errors(L):
    q = L.mx_quantize
    assert q(P, 1, 64, 64, 0, P, P, P, P, None) == ARG
    assert q(P, 1, 64, 64, 4, P, P, P, P, None) == ARG
    assert q(P, 1, 60, 64, 2, P, P, P, P, None) == SHAPE   # column blocks need rows % 32 == 0
    assert q(P, 1, 60, 64, 3, P, P, P, P, None) == SHAPE
    assert q(P, 1, 64, 60, 1, P, P, P, P, None) == SHAPE   # cols % 32 == 0 always
    assert q(P, 1, 64, 48, 2, P, P, P, P, None) == SHAPE
    assert q(P, -1, 64, 64, 1, P, P, P, P, None) == SHAPE
    assert q(P, 2 ** 40, 2 ** 20, 2 ** 20, 1, P, P, P, P, None) == SHAPE
    assert q(None, 1, 64, 64, 1, P, P, None, None, None) == NULL
    assert q(P, 1, 64, 64, 1, None, P, None, None, None) == NULL
    assert q(P, 1, 64, 64, 2, P, P, P, None, None) == NULL
    assert q(P8, 1, 64, 64, 1, P, P, None, None, None) == ALIGN
    assert q(P, 1, 64, 64, 3, P, P, P8, P, None) == ALIGN
    # empty problems are fine and launch nothing
    assert q(P, 0, 64, 64, 3, P, P, P, P, None) == OK
    assert q(P, 1, 0, 64, 1, P, P, None, None, None) == OK
    assert q(None, 1, 0, 64, 3, None, None, None, None, None) == OK  # empty: NULL allowed


def test_mx_dequantize_argument_errors(L):
    d = L.mx_dequantize
    assert d(P, P, 1, 64, 64, 3, P, None) == ARG
    assert d(P, P, 1, 64, 33, 1, P, None) == SHAPE
    assert d(P, P, 1, 60, 64, 2, P, None) == SHAPE
    assert d(None, P, 1, 64, 64, 1, P, None) == NULL
    assert d(P, None, 1, 64, 64, 2, P, None) == NULL
    assert d(P, P, 1, 64, 64, 1, P8, None) == ALIGN
    assert d(P, P, 1, 64, 0, 2, P, None) == OK
    assert d(None, None, 0, 64, 64, 1, None, None) == OK


def test_per_group_argument_errors(L):
    f = L.fp8_per_group_rowwise_quant
    assert f(P, 64, 64, P, 4, 2, P, P, None) == ARG
    assert f(P, 64, 60, P, 4, 0, P, P, None) == SHAPE
    assert f(P, -1, 64, P, 4, 0, P, P, None) == SHAPE
    assert f(P, 64, 64, P, 70000, 0, P, P, None) == SHAPE
    assert f(P, 64, 64, None, 4, 0, P, P, None) == NULL
    assert L.mxq_wait_timeouts(None) == NULL
    assert f(P, 64, 64, P, 4, 0, P, None, None) == NULL
    assert f(None, 64, 64, P, 4, 0, P, P, None) == NULL
    assert f(P, 64, 64, P, 4, 1, P8, P, None) == ALIGN
    assert f(P, 64, 64, P + 2, 4, 1, P, P, None) == ALIGN
    assert f(P, 64, 64, P, 0, 0, P, P, None) == OK  # no groups: nothing to write
    assert f(P, 64, 0, P, 4, 0, P, P, None) == OK   # no features


def test_encode_argument_errors(L):
    e = L.mx_e4m3_encode_f32
    assert e(P, -1, P, None) == SHAPE
    assert e(None, 16, P, None) == NULL
    assert e(P8, 16, P, None) == ALIGN
    assert e(P, 0, P, None) == OK


def test_binding_refuses_host_tensors():
    import torch
    x = torch.zeros(64, 64, dtype=torch.bfloat16)
    out = {k: torch.zeros(1, dtype=torch.uint8) for k in ("q_row", "s_row")}
    with pytest.raises(mxq.MxqError, match="CUDA tensor"):
        mxq.mx_quantize(x, mxq.ROW, **out)
    with pytest.raises(mxq.MxqError):
        mxq.fp8_per_group_rowwise_quant(x, torch.zeros(2, dtype=torch.int32), mxq.ROW_MAJOR,
                                        torch.zeros(64 * 64, dtype=torch.uint8),
                                        torch.zeros(2 * 64, dtype=torch.float32))


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(mxq, "_LIB", None)
    monkeypatch.setattr(mxq, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(mxq.MxqError, match="missing"):
        mxq.lib()


# ---- the per-group scheduler's host side (fp8_per_group_rowwise_plan) ----------------------

def _plan(M, K, G, layout, n_sm=148):
    return mxq.fp8_per_group_rowwise_plan(M, K, G, layout, n_sm=n_sm)


@pytest.mark.parametrize("M,K,G,layout,kernel,w,cl", [
    (65536, 5120, 16, 0, "tile", 64, 8),    # dispatch payload, row-major: 128-byte rows over 8 CTAs (73 KB tiles)
    (65536, 5120, 16, 1, "tile", 32, 8),    # column-major: 32-column slabs over 8 CTAs before 16 over 4
    (16640, 5120, 16, 0, "tile", 64, 4),
    (16640, 5120, 16, 1, "tile", 32, 2),
    (16640, 5120, 32, 0, "tile", 64, 1),    # one CTA of 128-byte rows up to 80 KB before a 2-CTA cluster
    (16640, 5120, 32, 1, "tile", 32, 1),
    (16640, 5120, 64, 1, "tile", 64, 1),
    (16640, 5120, 128, 0, "tile", 64, 1),
    (16640, 5120, 128, 1, "pair", 64, 1),   # two neighbouring groups per CTA
    (131072, 5120, 128, 1, "tile", 32, 2),  # the stress split: shaped by its average group
    (131072, 5120, 16, 0, "tile", 32, 8),   # 8192-row groups: 64-byte rows over 8 CTAs (70 KB tiles)
    (131072, 5120, 16, 1, "tile", 16, 8),
    (65536, 5120, 4, 0, "stream", 32, 1),   # 16384-row groups: too large for eight CTAs
    (65536, 5120, 4, 1, "stream", 32, 1),
    (64, 64, 0, 0, "none", 0, 0),
    (1000, 0, 4, 1, "none", 0, 0),
])
def test_per_group_plan_known_shapes(L, M, K, G, layout, kernel, w, cl):
    p = _plan(M, K, G, layout)
    assert (p["kernel"], p["slab_cols"], p["cluster"]) == (kernel, w, cl), p


def test_per_group_plan_invariants(L):
    import math
    for layout in (0, 1):
        for M in (1, 37, 1000, 16640, 65536, 131072, 1 << 20):
            for G in (1, 2, 3, 4, 16, 64, 128, 1000):
                n = (M + G - 1) // G
                p = _plan(M, 5120, G, layout)
                assert p["threads"] in (128, 256, 512)
                if p["kernel"] == "stream":
                    assert p["tile_rows"] == 0 and p["slab_cols"] == 32
                    # only when even eight CTAs of the narrowest slab cannot hold the average
                    # group (column-major tiles up to 48 KB, row-major 8-CTA tiles up to 80 KB)
                    w_min, cap = (16, 48 * 1024) if layout else (32, 80 * 1024)
                    assert math.ceil((n + 1.5 * math.sqrt(n)) / 8 + 48) * 2 * w_min > cap
                    continue
                w, cl, rows = p["slab_cols"], p["cluster"], p["tile_rows"]
                # a tile stays within 48 KB, or 80 KB for row-major single CTAs of 128-byte
                # rows and 8-CTA clusters
                big = layout == 0 and p["kernel"] == "tile" and (cl == 8 or (cl == 1 and w == 64))
                assert rows * 2 * w <= (80 if big else 48) * 1024
                assert rows % 16 == 0
                if p["kernel"] == "pair":
                    assert layout == 1 and G >= 2 and w == 64
                    assert rows >= 2 * n                     # both groups of a pair fit on average
                else:
                    assert cl in (1, 2, 4, 8) and w in ((16, 32, 64) if layout else (32, 64))
                    assert rows * cl >= n                    # the average group fits the cluster
    # the SM count changes only the streaming kernel's CTA size
    a, b = _plan(65536, 5120, 4, 0, n_sm=148), _plan(65536, 5120, 4, 0, n_sm=16)
    assert a["kernel"] == b["kernel"] == "stream" and a["threads"] >= b["threads"]


def test_per_group_plan_argument_errors(L):
    r = [ctypes.byref(ctypes.c_int()) for _ in range(5)]
    f = L.fp8_per_group_rowwise_plan
    assert f(64, 64, 4, 2, 148, *r) == ARG
    assert f(64, 60, 4, 0, 148, *r) == SHAPE
    assert f(64, 64, 70000, 0, 148, *r) == SHAPE
    assert f(-1, 64, 4, 0, 148, *r) == SHAPE
    assert f(64, 64, 4, 0, -1, *r) == SHAPE
    assert f(64, 64, 4, 0, 148, None, *r[1:]) == NULL
    assert f(64, 64, 4, 0, 0, *r) == OK   # 0: the current device's SM count (148 without one)
