"""The CPU oracle applied to independent slabs of a workload, for a process pool.

Test infrastructure.  MX blocks never cross a 32-row band (column blocks) or a row
(row blocks), and the per-group result of a feature depends only on that feature's
column, so the oracle's result on a row slab (MX, slab rows a multiple of 32) or a
column slab (per-group) is exactly that part of its result on the whole tensor.  The
functions here run in spawned worker processes: they import numpy and the oracle
only, never torch or the CUDA package.
"""
from __future__ import annotations

import multiprocessing
import os
from concurrent.futures import ProcessPoolExecutor

import numpy as np

import oracle


def mx_quantize_slab(x_bits: np.ndarray, axes: int):
    """Row slab (rows, cols) or (batch, rows, cols): MX quantize along `axes`."""
    return oracle.mx_quantize(x_bits, axes)


def mx_round_trip_slab(x_bits: np.ndarray):
    """Row slab (rows, cols): 1x32 and 32x1 quantize, then dequantize of the 1x32
    codes (the dispatch step's first two calls)."""
    rows, cols = x_bits.shape
    r = oracle.mx_quantize(x_bits, oracle.ROW | oracle.COL)
    r["y"] = oracle.mx_dequantize(r["q_row"], r["s_row"], 1, rows, cols, oracle.ROW)
    return r


def per_group_cols(x_bits: np.ndarray, offs: np.ndarray):
    """Column slab (M, k): per-group quantize, row-major codes and the slab's scales."""
    return oracle.per_group_quant(x_bits, offs, oracle.ROW_MAJOR)


def make_pool() -> ProcessPoolExecutor:
    """A pool over the host's cores.  Spawned, never forked: the parent has a CUDA
    context by the time the full-size tests run."""
    n = max(1, min(os.cpu_count() or 1, 32))
    return ProcessPoolExecutor(max_workers=n, mp_context=multiprocessing.get_context("spawn"))


def row_edges(rows: int, step: int) -> list[tuple[int, int]]:
    """[a, b) row slabs of `step` rows (step a multiple of 32)."""
    return [(a, min(rows, a + step)) for a in range(0, rows, step)]


def col_edges(cols: int, n: int) -> list[tuple[int, int]]:
    """About n [a, b) column slabs, each a multiple of 8 columns."""
    e = (np.linspace(0, cols // 8, n + 1).astype(int) * 8).tolist()
    e[-1] = cols
    return [(a, b) for a, b in zip(e[:-1], e[1:]) if b > a]


def mx_quantize_whole(pool, x_bits: np.ndarray, axes: int, step: int = 8192):
    """Oracle MX quantize of a whole (rows, cols) tensor, assembled from row slabs."""
    rows, cols = x_bits.shape
    edges = row_edges(rows, step)
    futs = [pool.submit(mx_quantize_slab, np.ascontiguousarray(x_bits[a:b]), axes) for a, b in edges]
    out = {}
    if axes & oracle.ROW:
        out["q_row"] = np.empty((rows, cols), np.uint8)
        out["s_row"] = np.empty((rows, cols // 32), np.uint8)
    if axes & oracle.COL:
        out["q_col"] = np.empty((cols, rows), np.uint8)
        out["s_col"] = np.empty((cols, rows // 32), np.uint8)
    for (a, b), f in zip(edges, futs):
        r = f.result()
        if axes & oracle.ROW:
            out["q_row"][a:b] = r["q_row"]
            out["s_row"][a:b] = r["s_row"]
        if axes & oracle.COL:
            out["q_col"][:, a:b] = r["q_col"]
            out["s_col"][:, a // 32:b // 32] = r["s_col"]
    return out


def per_group_whole(pool, x_bits: np.ndarray, offs: np.ndarray, n_slabs: int = 32):
    """Oracle per-group quantize of a whole (M, K) tensor (row-major codes, scales),
    assembled from column slabs."""
    M, K = x_bits.shape
    offs = np.ascontiguousarray(offs, dtype=np.int32)
    edges = col_edges(K, n_slabs)
    futs = [pool.submit(per_group_cols, np.ascontiguousarray(x_bits[:, a:b]), offs) for a, b in edges]
    q = np.empty((M, K), np.uint8)
    s = np.empty((offs.size, K), np.float32)
    for (a, b), f in zip(edges, futs):
        qa, sa = f.result()
        q[:, a:b] = qa
        s[:, a:b] = sa
    return q, s
