"""The CPU oracle run on all host cores, for the benchmark's CPU baseline.

TEST AND BASELINE INFRASTRUCTURE ONLY (like the rest of this package).  The oracle's
functions are used as they stand; this module only splits one step of the hot path
into independent slabs and runs them in a pool of spawned worker processes, with
inputs and outputs in shared memory so no slab is copied through a pipe:

  phase 1, row slabs (a multiple of 32 rows): MX quantize with 1x32 and 32x1 blocks,
           then dequantize of the 1x32 codes (MX blocks never cross a 32-row band);
  phase 2, column slabs (a multiple of 8 features): per-group quantize of the
           dequantized tokens (a feature's result depends only on its own column).
Each phase's slabs write disjoint parts of the outputs, so the result equals the
single-threaded oracle's on the whole batch.
"""
from __future__ import annotations

import multiprocessing
import os
from concurrent.futures import ProcessPoolExecutor
from multiprocessing import shared_memory

import numpy as np

from . import COL, ROW, ROW_MAJOR, mx_dequantize, mx_quantize, per_group_quant


def _attach(desc):
    name, shape, dt = desc
    shm = shared_memory.SharedMemory(name=name)
    return shm, np.ndarray(shape, np.dtype(dt), buffer=shm.buf)


def _rows_task(descs: dict, a: int, b: int) -> None:
    shms, arr = [], {}
    for k, d in descs.items():
        shm, arr[k] = _attach(d)
        shms.append(shm)
    try:
        x = np.ascontiguousarray(arr["x"][a:b])
        rows, cols = x.shape
        r = mx_quantize(x, ROW | COL)
        arr["q_row"][a:b] = r["q_row"]
        arr["s_row"][a:b] = r["s_row"]
        arr["q_col"][:, a:b] = r["q_col"]
        arr["s_col"][:, a // 32:b // 32] = r["s_col"]
        arr["y"][a:b] = mx_dequantize(r["q_row"], r["s_row"], 1, rows, cols, ROW)
    finally:
        del arr
        for shm in shms:
            shm.close()


def _cols_task(descs: dict, offs: np.ndarray, a: int, b: int) -> None:
    shms, arr = [], {}
    for k, d in descs.items():
        shm, arr[k] = _attach(d)
        shms.append(shm)
    try:
        q, s = per_group_quant(np.ascontiguousarray(arr["y"][:, a:b]), offs, ROW_MAJOR)
        arr["q"][:, a:b] = q
        arr["scales"][:, a:b] = s
    finally:
        del arr
        for shm in shms:
            shm.close()


def _noop(_i: int = 0) -> int:
    return os.getpid()


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class StepOnAllCores:
    """One step of the hot path (MX dual-axis quantize -> dequantize -> per-group
    row-major) by the oracle on `x_bits` (rows, cols), spread over `workers`
    processes.  Create once (allocates shared memory, starts and warms the pool), call
    run() to time, close() when done."""

    def __init__(self, x_bits: np.ndarray, offs: np.ndarray, workers: int | None = None):
        rows, cols = x_bits.shape
        assert rows % 32 == 0 and cols % 32 == 0
        self.rows, self.cols = rows, cols
        self.offs = np.minimum(np.asarray(offs, np.int64), rows).astype(np.int32)
        self.workers = workers or host_cores()
        shapes = {"x": ((rows, cols), np.uint16), "q_row": ((rows, cols), np.uint8),
                  "s_row": ((rows, cols // 32), np.uint8), "q_col": ((cols, rows), np.uint8),
                  "s_col": ((cols, rows // 32), np.uint8), "y": ((rows, cols), np.uint16),
                  "q": ((rows, cols), np.uint8), "scales": ((self.offs.size, cols), np.float32)}
        self._shm, self.arr, self.descs = {}, {}, {}
        for k, (shape, dt) in shapes.items():
            n = int(np.prod(shape)) * np.dtype(dt).itemsize
            shm = shared_memory.SharedMemory(create=True, size=max(n, 1))
            self._shm[k] = shm
            self.arr[k] = np.ndarray(shape, dt, buffer=shm.buf)
            self.descs[k] = (shm.name, shape, np.dtype(dt).str)
        self.arr["x"][...] = x_bits
        self.pool = ProcessPoolExecutor(max_workers=self.workers,
                                        mp_context=multiprocessing.get_context("spawn"))
        list(self.pool.map(_noop, range(4 * self.workers)))  # every worker started
        # slabs: about four per worker and phase
        n_row = max(1, min(rows // 32, 4 * self.workers))
        e = np.linspace(0, rows // 32, n_row + 1).astype(int) * 32
        self.row_slabs = [(int(a), int(b)) for a, b in zip(e[:-1], e[1:]) if b > a]
        n_col = max(1, min(cols // 8, 4 * self.workers))
        e = np.linspace(0, cols // 8, n_col + 1).astype(int) * 8
        self.col_slabs = [(int(a), int(b)) for a, b in zip(e[:-1], e[1:]) if b > a]

    def run(self) -> None:
        descs = self.descs
        for f in [self.pool.submit(_rows_task, descs, a, b) for a, b in self.row_slabs]:
            f.result()
        for f in [self.pool.submit(_cols_task, descs, self.offs, a, b) for a, b in self.col_slabs]:
            f.result()

    def close(self) -> None:
        self.pool.shutdown()
        self.arr.clear()
        for shm in self._shm.values():
            shm.close()
            shm.unlink()
        self._shm.clear()
