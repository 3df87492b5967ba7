"""Benchmark of the MXFP8 / per-group FP8 quantization hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload: the MXFP8 dispatch payload of the Llama4 debug configuration on the
torchtitan mxfp8 all-to-all page -- (local batch 8 x seq 8192, dim 5120) bf16 tokens,
rows N(0,1) times a per-row lognormal scale, 0.1% outliers x100, routed to 16 experts
with multinomial-uniform group sizes.  One step is one pass of the whole hot path
over that batch:
  1. mx_quantize, 1x32 and 32x1 blocks from one read (dispatch payload + the
     column-blocked copy the backward pass needs),
  2. mx_dequantize of the 1x32 payload back to bf16 (receive side of the all-to-all),
  3. fp8_per_group_rowwise_quant of the received tokens, 16 groups, row-major E4M3
     (left operand of the scaled grouped GEMM).
Metric: GB/s of algorithmic bytes (read + written) per step, and the fraction of the
measured HBM bandwidth.  Inputs (671 MB) are larger than L2 (126 MB), so no L2 flush
is inserted between steps.  With N GPUs (torchrun), every rank processes its own
batch (weak scaling, no collective on the data path); the step time is the max over
ranks and ``value`` counts the bytes of all ranks.

``--impl reference`` times the CPU oracle (the plain C reference the tests use) on
bounded samples of the same workload on the host cores, rank 0 only.

``--configs`` (1 GPU) instead times every hot-path call at each workload
configuration -- the per-group (16640, 5120) tensor with 16..128 groups in both
layouts, the dual-axis activations and expert weights, the stress mix, and the
dispatch payload's three calls -- and prints one JSON line per case.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import platform
import re
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

ROWS, COLS, N_GROUPS = 65536, 5120, 16
METRIC = "quant GB/s (bytes read+written) and % of B200 HBM peak, 1 GPU"
UNIT = "GB/s"
WORKLOAD = ("MXFP8 dispatch payload (65536, 5120) bf16 = local_bs 8 x seq 8192 x dim 5120, "
            "16 experts: MX dual-axis quantize -> MX dequantize -> per-group FP8 rowwise "
            "(row-major)")


def workload_name(rows: int, groups: int) -> str:
    """The workload string for the timed step; other sizes than the dispatch payload's
    (smaller cases for profiling) are named by their own shape."""
    if rows == ROWS and groups == N_GROUPS:
        return WORKLOAD
    return (f"MXFP8 dispatch-payload recipe at ({rows}, {COLS}) bf16, {groups} experts: MX dual-axis "
            "quantize -> MX dequantize -> per-group FP8 rowwise (row-major)")
FALLBACK_HBM_GBS = 6650.0


# ---- algorithmic bytes --------------------------------------------------------------------

def alg_bytes(rows: int, cols: int, groups: int) -> dict:
    n = rows * cols
    return {
        "mx_quantize_dual": 2 * n + 2 * (n + n // 32),   # read bf16, write 2 x (E4M3 + E8M0)
        "mx_dequantize": n + n // 32 + 2 * n,            # read E4M3 + E8M0, write bf16
        "per_group_quant": 3 * n + 4 * groups * cols + 4 * groups,  # X once, q, scales, offsets
    }


# The source files each timed call's kernels (and their launch code) are built from.
KERNEL_SOURCES = {
    "mx_quantize_dual": ["mx_quant.cu", "mxq_device.cuh"],
    "mx_dequantize": ["mx_dequant.cu", "mxq_device.cuh"],
    "per_group_quant": ["per_group.cu", "mxq_device.cuh", "tensor_map.cu"],
}


def _code_only(text: str) -> str:
    """Source text without comments and blank lines (a comment edit keeps the hash)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines if ln)


def sources_sha(kernel: str | None = None) -> str:
    """Hash of a call's kernel sources, comments aside (all of csrc/ when kernel is
    None)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mxfp8_quantization_moe_mx_b200", "csrc")
    names = KERNEL_SOURCES[kernel] if kernel else sorted(os.listdir(csrc))
    for name in names:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode())
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def recorded_traffic(kernel: str):
    """dram bytes per launch from the committed ncu summary, if it was taken on the
    current sources of that call's kernels (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    ent = rec.get(kernel)
    if not ent or ent.get("sources_sha") != sources_sha(kernel):
        return None
    return ent.get("dram_bytes_per_launch")


# ---- clocks -----------------------------------------------------------------------------------

def nvml_handle(pynvml, device_index: int):
    """The NVML handle of CUDA device `device_index` of this process, matched by PCI
    location (NVML numbers every GPU of the machine, CUDA only the visible ones)."""
    p = torch.cuda.get_device_properties(device_index)
    for i in range(pynvml.nvmlDeviceGetCount()):
        h = pynvml.nvmlDeviceGetHandleByIndex(i)
        pci = pynvml.nvmlDeviceGetPciInfo(h)
        if (pci.domain, pci.bus, pci.device) == (p.pci_domain_id, p.pci_bus_id, p.pci_device_id):
            return h
    return pynvml.nvmlDeviceGetHandleByIndex(device_index)


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read-only) every 2 ms, with
    the host time of each sample, so that even a timed region of ~10 ms gets several.
    A failed NVML read is counted and sampling goes on.  `region(t0, t1)` marks the timed
    region; if fewer than three samples fall inside it, the summary uses the samples
    taken right after it, while the caller keeps the GPU under the same load (untimed
    steps), and says so in `window`."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int):
        self.samples, self.masks = [], []  # (host time, SM MHz), (host time, reason mask)
        self.max_mhz, self.errors, self.last_error = None, 0, None
        self.t0 = self.t1 = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = nvml_handle(pynvml, device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._reasons = (getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None)
                             or getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
            self._ok = True
        except Exception as e:
            self.last_error = repr(e)

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            t = time.perf_counter()
            try:
                self.samples.append((t, nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)))
            except Exception as e:
                self.errors += 1
                self.last_error = repr(e)
            if self._reasons is not None:
                try:
                    self.masks.append((t, self._reasons(self._h)))
                except Exception as e:
                    self.errors += 1
                    self.last_error = repr(e)
            time.sleep(0.002)

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
            # the first NVML reads can be slow: wait for one sample (at most 1 s)
            t0 = time.perf_counter()
            while not self.samples and not self.errors and time.perf_counter() - t0 < 1.0:
                time.sleep(0.005)
        return self

    def region(self, t0: float, t1: float):
        self.t0, self.t1 = t0, t1

    def __exit__(self, *a):
        if self._ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        rec = {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
               "window": "timed region"}
        if self.errors or not self._ok:
            rec["nvml_errors"] = self.errors
            rec["nvml_last_error"] = self.last_error
        if not self._ok or self.t0 is None:
            return rec

        def pick(lo, hi):
            return ([m for t, m in self.samples if lo <= t <= hi], [k for t, k in self.masks if lo <= t <= hi])

        mhz, masks = pick(self.t0, self.t1)
        if len(mhz) < 3:
            after, after_masks = pick(self.t1, float("inf"))
            if len(after) >= 3:
                mhz, masks = mhz + after, masks + after_masks
                rec["window"] = "timed region + the untimed steps right after it (same load)"
        reasons = set()
        for k in masks:
            reasons |= {name for bit, name in self.REASONS.items() if k & bit}
        rec.update({"sm_mhz": float(np.median(mhz)) if mhz else None, "reasons": sorted(reasons - {"gpu_idle"}),
                    "samples": len(mhz)})
        return rec


# ---- distributed plumbing ------------------------------------------------------------------------

def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def rank_seed(rank: int) -> int:
    from mxfp8_quantization_moe_mx_b200 import workloads as wl
    return wl.SEED_BASE + 1 + 1000 * rank


# ---- CPU oracle timing ------------------------------------------------------------------------------

def oracle_step_on_sample(xb: np.ndarray, offs: np.ndarray, rows: int):
    """One pass of the three operations of a step by the CPU oracle, on the first
    `rows` rows of the batch (offsets clipped to them).  Returns algorithmic bytes."""
    import oracle
    sub = np.ascontiguousarray(xb[:rows])
    r = oracle.mx_quantize(sub, oracle.ROW | oracle.COL)
    y = oracle.mx_dequantize(r["q_row"], r["s_row"], 1, rows, sub.shape[1], oracle.ROW)
    o = np.minimum(offs, rows).astype(np.int32)
    oracle.per_group_quant(y, o, oracle.ROW_MAJOR)
    return sum(alg_bytes(rows, sub.shape[1], len(offs)).values())


def time_oracle(xb, offs, rows, steps, warmup):
    for _ in range(warmup):
        oracle_step_on_sample(xb, offs, rows)
    t0 = time.perf_counter()
    total = 0
    for _ in range(steps):
        total += oracle_step_on_sample(xb, offs, rows)
    dt = time.perf_counter() - t0
    return total / dt / 1e9, dt


def cpu_baseline(x_host, offs_host, args) -> dict:
    """The oracle timed on the host: the whole batch on every core, and the first
    `cpu_rows` rows single-threaded.  `value` is the all-cores figure."""
    from oracle.parallel import StepOnAllCores, host_cores
    xb = x_host.view(torch.int16).numpy().view(np.uint16)
    offs = offs_host.numpy()
    M, K = xb.shape
    G = offs.size
    rows1 = min(args.cpu_rows, M)
    v1, dt1 = time_oracle(xb, offs, rows1, steps=1, warmup=0)
    cores = host_cores()
    # the shared-memory arrays of the all-cores run take about 7.1 bytes per element;
    # use at most half of /dev/shm (the whole batch when it fits)
    try:
        import shutil
        free = shutil.disk_usage("/dev/shm").free
    except Exception:
        free = 0
    rows = min(M, int(free * 0.5 / (7.1 * K)) // 32 * 32)
    if rows < 32:
        return {"value": round(v1, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
                "sample": f"first {rows1} of {M} rows (offsets clipped), one pass of the three ops, "
                          f"{dt1:.1f} s single-threaded (no room in /dev/shm for the all-cores run)",
                "cpu": cpu_info(), "host_cpus": os.cpu_count()}
    runner = StepOnAllCores(np.ascontiguousarray(xb[:rows]), offs, workers=cores)
    try:
        t0 = time.perf_counter()
        runner.run()
        dt = time.perf_counter() - t0
    finally:
        runner.close()
    vall = sum(alg_bytes(rows, K, G).values()) / dt / 1e9
    what = "the whole batch" if rows == M else f"the first {rows} of {M} rows (offsets clipped)"
    return {"value": round(vall, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": (f"one step over {what} ({K} features, {G} groups) on {cores} worker processes: "
                       f"row slabs for MX quantize/dequantize, column slabs for per-group; {dt:.1f} s"),
            "single_thread": {"value": round(v1, 4), "unit": UNIT, "cores": 1,
                              "sample": f"first {rows1} of {M} rows (offsets clipped), one pass of the three ops, "
                                        f"{dt1:.1f} s"},
            "cpu": cpu_info(), "host_cpus": os.cpu_count()}


def cpu_info():
    model = platform.processor() or ""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except Exception:
        pass
    return model


# ---- our arm ----------------------------------------------------------------------------------------------

def run_ours(args, world, rank, local):
    import mxfp8_quantization_moe_mx_b200 as mxq
    from mxfp8_quantization_moe_mx_b200 import workloads as wl

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the product path has no CPU fallback)")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    mxq.lib()

    t = wl.dispatch(seed=rank_seed(rank), rows=args.rows, cols=COLS, n_groups=args.groups)
    x_host, offs_host = t["x"], t["offs"]
    x = x_host.to(dev)
    offs = offs_host.to(dev)
    M, K = x.shape
    out = mxq.empty_mx_outputs(x, mxq.ROW | mxq.COL)
    y = torch.empty_like(x)
    q = torch.empty(M, K, dtype=torch.uint8, device=dev)
    sc = torch.empty(args.groups, K, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    names = ["mx_quantize_dual", "mx_dequantize", "per_group_quant"]

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        mxq.mx_quantize(x, mxq.ROW | mxq.COL, **out, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        mxq.mx_dequantize(out["q_row"], out["s_row"], 1, M, K, mxq.ROW, y, stream=stream)
        if ev is not None:
            ev[2].record(stream)
        mxq.fp8_per_group_rowwise_quant(y, offs, mxq.ROW_MAJOR, q, sc, stream=stream)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        t0 = time.perf_counter()
        start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        stop.record(stream)
        torch.cuda.synchronize(dev)
        clocks.region(t0, time.perf_counter())
        # untimed steps under the same load: clock samples for a region too short to get three
        for _ in range(args.steps):
            step()
        torch.cuda.synchronize(dev)
    barrier(world)
    ms_total = start.elapsed_time(stop)
    per_kernel_ms = {n: float(np.mean([evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(args.steps)]))
                     for j, n in enumerate(names)}
    ms_step = max_over_ranks(ms_total / args.steps, world, dev)

    ab = alg_bytes(M, K, args.groups)
    bytes_step = sum(ab.values())
    value = world * bytes_step / (ms_step * 1e-3) / 1e9
    peak, peak_src = hbm_peak()
    dom = max(names, key=lambda n: per_kernel_ms[n])
    achieved = ab[dom] / (per_kernel_ms[dom] * 1e-3) / 1e9
    kernels = {n: {"ms": round(per_kernel_ms[n], 5), "alg_bytes": ab[n],
                   "GB_s": round(ab[n] / (per_kernel_ms[n] * 1e-3) / 1e9, 1),
                   "frac_of_hbm": round(ab[n] / (per_kernel_ms[n] * 1e-3) / 1e9 / peak, 4)}
               for n in names}

    # ---- end to end through the public API with host buffers: every step uploads its
    # input from pinned host memory and reads every output back.  Steps are pipelined
    # over two device slots and three streams (upload, compute, download), so the
    # upload of one step overlaps the download of the previous one on the full-duplex
    # link; events keep each slot's upload, compute and download in order.
    e2e = None
    if not args.no_e2e:
        e2e_steps = max(2, min(args.steps, args.e2e_steps))
        xh = x_host.pin_memory()
        oh = offs_host.pin_memory()
        slots = []
        for k in range(2):
            xs = x if k == 0 else torch.empty_like(x)
            os_ = offs if k == 0 else torch.empty_like(offs)
            o = out if k == 0 else mxq.empty_mx_outputs(x, mxq.ROW | mxq.COL)
            ys = y if k == 0 else torch.empty_like(y)
            qs = q if k == 0 else torch.empty_like(q)
            ss = sc if k == 0 else torch.empty_like(sc)
            slots.append({"x": xs, "offs": os_, "out": o, "y": ys, "q": qs, "sc": ss,
                          "dev_outs": [o["q_row"], o["s_row"], o["q_col"], o["s_col"], ys, qs, ss]})
        outs_host = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in slots[0]["dev_outs"]]
        h2d = xh.numel() * xh.element_size() + oh.numel() * oh.element_size()
        d2h = sum(o.numel() * o.element_size() for o in slots[0]["dev_outs"])
        s_up, s_dn = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()
        last_compute = [None, None]   # per slot: compute finished (inputs free for reuse)
        last_download = [None, None]  # per slot: download finished (outputs free for reuse)

        def e2e_step(i):
            k = i % 2
            sl = slots[k]
            with torch.cuda.stream(s_up):
                if last_compute[k] is not None:
                    s_up.wait_event(last_compute[k])
                sl["x"].copy_(xh, non_blocking=True)
                sl["offs"].copy_(oh, non_blocking=True)
                up = ev()
                up.record(s_up)
            stream.wait_event(up)
            if last_download[k] is not None:
                stream.wait_event(last_download[k])
            M_, K_ = sl["x"].shape
            mxq.mx_quantize(sl["x"], mxq.ROW | mxq.COL, **sl["out"], stream=stream)
            mxq.mx_dequantize(sl["out"]["q_row"], sl["out"]["s_row"], 1, M_, K_, mxq.ROW, sl["y"], stream=stream)
            mxq.fp8_per_group_rowwise_quant(sl["y"], sl["offs"], mxq.ROW_MAJOR, sl["q"], sl["sc"], stream=stream)
            done = ev()
            done.record(stream)
            last_compute[k] = done
            with torch.cuda.stream(s_dn):
                s_dn.wait_event(done)
                for hd, dd in zip(outs_host, sl["dev_outs"]):
                    hd.copy_(dd, non_blocking=True)
                dn = ev()
                dn.record(s_dn)
            last_download[k] = dn

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_up)
        for i in range(e2e_steps):
            e2e_step(i)
        e1.record(s_dn)
        torch.cuda.synchronize(dev)
        barrier(world)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world, dev)
        e2e = {"value": round(world * bytes_step / (e2e_ms * 1e-3) / 1e9, 2), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 3),
               "steps": e2e_steps,
               "note": ("pinned host input -> 3 library calls -> every output copied back to pinned host "
                        "memory; steps pipelined over two device slots (upload / compute / download streams)")}

    # ---- CPU oracle baseline on a bounded sample (rank 0, N = 1 only)
    # ---- every call at every workload configuration (1 GPU): the per-configuration
    # figures, L2 flushed between timed iterations
    configs = None
    if rank == 0 and world == 1 and not args.no_configs:
        configs = time_configs(dev, iters=args.config_iters, warmup=max(3, args.warmup))

    # ---- CPU oracle baseline on a bounded sample (rank 0, N = 1 only): the oracle as
    # it stands, on every host core (slabs in a spawned process pool) over the whole
    # batch, and single-threaded on the first rows
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(x_host, offs_host, args)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16->e4m3/e8m0",
            "data": "synthetic (seeded; per-rank batch)",
            "config": {"workload": workload_name(M, args.groups), "rows": M, "cols": K, "groups": args.groups,
                       "global_batch_rows": world * M, "l2": "inputs larger than L2 (671 MB > 126 MB), no flush",
                       "parallelism": f"replicas x{world}"},
            "frac_of_hbm": round(value / world / peak, 4),
            "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1), "peak": peak,
                         "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "traffic": recorded_traffic(dom), "peak_source": peak_src,
                         "alg_bytes_per_launch": ab[dom]},
            "kernels": kernels,
            "gpu_launches": 3 * args.steps,
            "clocks": clocks.summary(),
            "e2e": e2e,
            "cpu_baseline": cpu,
            "configs": configs,
        }
        print(json.dumps(line), flush=True)


# ---- reference arm: the CPU oracle --------------------------------------------------------------------------

class L2Flush:
    """Between timed iterations: write a 256 MB buffer (evicts whatever the last call
    left in L2), then read another 256 MB buffer, so the dirty lines of the write are
    written back before the next timed call starts instead of during it.  The timed
    call then starts with a cold, clean L2 (126 MB on B200)."""

    def __init__(self, dev):
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.r = torch.ones(256 << 18, dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.fill_(1)
        self.r.sum()


def fp8_peak():
    """The fp8 dense tensor peak: the measured bf16 burst figure times the nominal
    fp8 / bf16 ratio (4.5 / 2.25 PFLOP/s)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return 2.0 * float(json.load(f)["bf16_tflops"]), "measured bf16 burst x 2 (nominal fp8/bf16 ratio)"
    except Exception:
        return 2.0 * 1590.0, "fallback bf16 x 2"


def time_configs(dev, iters: int, warmup: int, only: str | None = None, gemm_rows: int = 65536):
    """Every hot-path call at every workload configuration: device time with CUDA
    events on the launching stream, the L2 flushed (outside the events) before each
    timed iteration, median over `iters`.  Returns one record per (configuration, call)
    with microseconds, algorithmic GB/s and the fraction of the measured HBM
    bandwidth."""
    import mxfp8_quantization_moe_mx_b200 as mxq
    from mxfp8_quantization_moe_mx_b200 import workloads as wl

    stream = torch.cuda.current_stream(dev)
    peak, _ = hbm_peak()
    flush = L2Flush(dev)
    recs = []

    def timed(fn):
        for _ in range(warmup):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
        for e0, e1 in ev:
            flush()
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = sorted(e0.elapsed_time(e1) for e0, e1 in ev)
        return float(np.median(ms)), ms[0]

    def want(config, call, groups=None):
        if only is None:
            return True
        key = f"{config} | {call}" + (f" | groups={groups}" if groups is not None else "")
        return only in key

    def emit(config, call, nbytes, ms_pair, **extra):
        if ms_pair is None:
            return
        ms, ms_min = ms_pair
        gbs = nbytes / (ms * 1e-3) / 1e9
        recs.append({"config": config, "call": call, "us": round(ms * 1e3, 2), "us_min": round(ms_min * 1e3, 2),
                     "alg_bytes": nbytes, "GB_s": round(gbs, 1), "frac_of_hbm": round(gbs / peak, 4), **extra})

    if only is not None and "grouped_gemm" in only:
        gemm_case(dev, stream, timed, recs, gemm_rows)
        return recs

    def mx_cases(config, x):
        b, r, c = (1, *x.shape) if x.dim() == 2 else tuple(x.shape)
        n = b * r * c
        for axes, name, per in ((mxq.ROW, "mx_quantize 1x32", 3.03125), (mxq.COL, "mx_quantize 32x1", 3.03125),
                                (mxq.ROW | mxq.COL, "mx_quantize dual", 4.0625)):
            if not want(config, name):
                continue
            out = mxq.empty_mx_outputs(x, axes)
            emit(config, name, int(per * n), timed(lambda: mxq.mx_quantize(x, axes, **out, stream=stream)))
            del out
        for axis, name in ((mxq.ROW, "mx_dequantize 1x32"), (mxq.COL, "mx_dequantize 32x1")):
            if not want(config, name):
                continue
            out = mxq.empty_mx_outputs(x, axis)
            mxq.mx_quantize(x, axis, **out, stream=stream)
            q, s = (out["q_row"], out["s_row"]) if axis == mxq.ROW else (out["q_col"], out["s_col"])
            y = torch.empty_like(x)
            emit(config, name, int(3.03125 * n), timed(lambda: mxq.mx_dequantize(q, s, b, r, c, axis, y, stream=stream)))
            del out, y

    def pg_cases(config, x, offs, layouts=(mxq.ROW_MAJOR, mxq.COL_MAJOR)):
        M, K = x.shape
        G = offs.numel()
        q = torch.empty(M * K, dtype=torch.uint8, device=dev)
        sc = torch.empty(G * K, dtype=torch.float32, device=dev)
        for layout in layouts:
            name = "fp8_per_group_rowwise_quant " + ("row-major" if layout == mxq.ROW_MAJOR else "col-major")
            if not want(config, name, G):
                continue
            emit(config, name, 3 * M * K + 4 * G * K + 4 * G,
                 timed(lambda: mxq.fp8_per_group_rowwise_quant(x, offs, layout, q, sc, stream=stream)), groups=G)

    t = wl.dispatch()
    x = t["x"].to(dev)
    mx_cases("dispatch (65536, 5120)", x)
    pg_cases("dispatch (65536, 5120), 16 experts", x, t["offs"].to(dev))
    del x, t
    for G in (16, 32, 64, 128):
        t = wl.per_group(n_groups=G)
        pg_cases("per-group (16640, 5120)", t["x"].to(dev), t["offs"].to(dev))
        del t
    # layouts for the scaled grouped GEMM: column-major per-group codes (5120, 16640)
    # -> row-major, and the dispatch payload's E8M0 scales -> 128 x 4 tiles per expert
    src = torch.randint(0, 256, (5120, 16640), dtype=torch.uint8, device=dev)
    dst = torch.empty_like(src)
    cfg_t, call_t = "per-group codes (5120, 16640) column-major", "mxq_transpose_u8 -> row-major"
    emit(cfg_t, call_t, 2 * src.numel(),
         timed(lambda: mxq.mxq_transpose_u8(src, dst, stream=stream)) if want(cfg_t, call_t) else None)
    del src, dst
    t = wl.dispatch(rows=65536, cols=32)
    sc = torch.randint(0, 256, (65536, 160), dtype=torch.uint8, device=dev)
    od = t["offs"].to(dev)
    nb = mxq.mx_scales_blocked_bytes(1, 65536, 160, od.numel())
    blk = torch.empty(nb, dtype=torch.uint8, device=dev)
    used = sum(-(-int(n) // 128) * 128 for n in np.diff(np.concatenate([[0], t["offs"].numpy()]))) * 160
    cfg_b, call_b = "dispatch E8M0 scales (65536, 160), 16 experts", "mx_scales_to_blocked"
    emit(cfg_b, call_b, sc.numel() + used,
         timed(lambda: mxq.mx_scales_to_blocked(sc, blk, od, stream=stream)) if want(cfg_b, call_b) else None)
    del sc, blk, od, t
    t = wl.dual_axis()
    mx_cases("dual-axis activations (16384, 5120)", t["act"].to(dev))
    w = t["w"].to(dev)
    mx_cases("dual-axis expert weights (16, 8192, 5120)", w)
    # the 3-D left operand: every expert matrix its own group
    E, R, C = w.shape
    qw = torch.empty(w.numel(), dtype=torch.uint8, device=dev)
    sw = torch.empty(E * C, dtype=torch.float32, device=dev)
    for layout in (mxq.ROW_MAJOR, mxq.COL_MAJOR):
        cfg_w = "expert weights (16, 8192, 5120), one group per expert"
        call_w = "fp8_per_group_rowwise_quant_batched " + ("row-major" if layout == mxq.ROW_MAJOR else "col-major")
        if not want(cfg_w, call_w, E):
            continue
        emit(cfg_w, call_w, 3 * w.numel() + 4 * E * C,
             timed(lambda: mxq.fp8_per_group_rowwise_quant_batched(w, layout, qw, sw, stream=stream)), groups=E)
    del t, w, qw, sw
    t = wl.stress()
    x = t["x"].to(dev)
    pg_cases("stress (131072, 5120), 128 Zipf groups, 20 empty", x, t["offs"].to(dev), layouts=(mxq.COL_MAJOR,))
    mx_cases("stress (131072, 5120)", x)
    del x, t
    torch.cuda.empty_cache()
    if want("MoE expert GEMM", "mx_grouped_gemm"):
        gemm_case(dev, stream, timed, recs, gemm_rows)
    del flush
    torch.cuda.empty_cache()
    return recs


def gemm_case(dev, stream, timed, recs, rows: int = 65536):
    """The consumer of the dispatch payload: the MXFP8 grouped GEMM of the tokens
    (rows, 5120) with 16 expert matrices (8192, 5120) (the Llama4 debug model's
    expert shape), every operand quantized and its scales laid out by this library.
    Reported in TFLOP/s (2 M N K) against the fp8 tensor peak."""
    import mxfp8_quantization_moe_mx_b200 as mxq
    from mxfp8_quantization_moe_mx_b200 import workloads as wl

    G, N, K = 16, 8192, 5120
    t = wl.dispatch(rows=rows, cols=K, n_groups=G)
    x, offs = t["x"].to(dev), t["offs"].to(dev)
    w = wl.dual_axis(act_rows=32, dim=K, experts=G, hidden=N)["w"].to(dev)
    qa = mxq.empty_mx_outputs(x, mxq.ROW)
    qb = mxq.empty_mx_outputs(w, mxq.ROW)
    mxq.mx_quantize(x, mxq.ROW, **qa, stream=stream)
    mxq.mx_quantize(w, mxq.ROW, **qb, stream=stream)
    sfa = torch.empty(mxq.mx_scales_blocked_bytes(1, rows, K // 32, G), dtype=torch.uint8, device=dev)
    sfb = torch.empty(mxq.mx_scales_blocked_bytes(G, N, K // 32, 0), dtype=torch.uint8, device=dev)
    mxq.mx_scales_to_blocked(qa["s_row"][0], sfa, offs, stream=stream)
    mxq.mx_scales_to_blocked(qb["s_row"], sfb, stream=stream)
    del x, w
    out = torch.empty(rows, N, dtype=torch.bfloat16, device=dev)
    ms, ms_min = timed(lambda: mxq.mx_grouped_gemm(qa["q_row"][0], sfa, qb["q_row"], sfb, offs, out, stream=stream))
    flops = 2.0 * rows * N * K
    tf = flops / (ms * 1e-3) / 1e12
    pk, src = fp8_peak()
    recs.append({"config": f"MoE expert GEMM: tokens ({rows}, {K}) x 16 experts ({N}, {K}), 16 groups",
                 "call": "mx_grouped_gemm", "us": round(ms * 1e3, 2), "us_min": round(ms_min * 1e3, 2),
                 "flops": flops, "TFLOP_s": round(tf, 1), "frac_of_fp8_peak": round(tf / pk, 4),
                 "fp8_peak_tflops": pk, "peak_source": src})
    del qa, qb, sfa, sfb, out, offs


def run_configs(args):
    """`--configs`: the per-configuration records, one JSON line each."""
    import mxfp8_quantization_moe_mx_b200 as mxq

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the product path has no CPU fallback)")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    mxq.lib()
    for r in time_configs(dev, iters=max(5, min(args.steps, 50)), warmup=args.warmup, only=args.filter,
                          gemm_rows=args.gemm_rows):
        print(json.dumps(r), flush=True)


def run_reference(args, world, rank, local):
    if rank != 0:
        return
    from mxfp8_quantization_moe_mx_b200 import workloads as wl
    rows = min(args.ref_rows, args.rows)
    t = wl.dispatch(seed=rank_seed(0), rows=args.rows, cols=COLS, n_groups=args.groups)
    xb = t["x"].view(torch.int16).numpy().view(np.uint16)
    offs = t["offs"].numpy()
    v, dt = time_oracle(xb, offs, rows, steps=args.steps, warmup=args.warmup)
    ms = dt / args.steps * 1e3
    sample = f"first {rows} of {args.rows} rows per step (offsets clipped), single-threaded plain C oracle"
    line = {
        "impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16->e4m3/e8m0",
        "data": "synthetic (seeded)",
        "config": {"workload": workload_name(args.rows, args.groups), "rows": args.rows, "cols": COLS,
                   "groups": args.groups,
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": round(v, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample, "cpu": cpu_info()},
        "e2e": {"value": round(v, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=32768)
    ap.add_argument("--ref-rows", type=int, default=512)
    ap.add_argument("--groups", type=int, default=N_GROUPS,
                    help="expert groups of the per-group step (default 16)")
    ap.add_argument("--rows", type=int, default=ROWS,
                    help="token rows of the workload (default: the dispatch payload's 65536)")
    ap.add_argument("--no-configs", action="store_true",
                    help="leave out the per-configuration timings of the default run")
    ap.add_argument("--config-iters", type=int, default=10,
                    help="timed iterations per configuration and call (L2 flushed before each)")
    ap.add_argument("--filter", default=None,
                    help="with --configs: only the calls whose name contains this (grouped_gemm: the GEMM alone)")
    ap.add_argument("--gemm-rows", type=int, default=65536,
                    help="token rows of the grouped-GEMM configuration (default: the dispatch payload's)")
    ap.add_argument("--configs", action="store_true",
                    help="time every hot-path call at every workload configuration (1 GPU)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.configs:
        run_configs(args)
        return
    if args.impl == "reference":
        # host-only: rank 0 times the oracle, the other ranks exit without work
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank, 0)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
