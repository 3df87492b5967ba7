"""Host-side logic of bench.py without a GPU: algorithmic byte counts, the two-rank
(gloo, world size 2) barrier / max-over-ranks used for multi-GPU timing, the reference
arm's per-rank behaviour under a torchrun-style environment, and the bookkeeping that
ties recorded ncu traffic to the kernel sources it was taken on."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_algorithmic_bytes_per_element():
    n_rows, n_cols, g = 64, 96, 4
    ab = bench.alg_bytes(n_rows, n_cols, g)
    n = n_rows * n_cols
    assert ab["mx_quantize_dual"] == pytest.approx(4.0625 * n)
    assert ab["mx_dequantize"] == pytest.approx(3.03125 * n)
    assert ab["per_group_quant"] == 3 * n + 4 * g * n_cols + 4 * g


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        m = bench.max_over_ranks(1.5 + rank, world, torch.device("cpu"))
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.rank_seed(rank))
        q.put((rank, m, seeds))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_over_ranks_gloo():
    world, port = 2, 29611
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, seeds in res:
        assert m == 2.5                      # the slowest rank's time
        assert len(set(seeds)) == world      # each rank its own batch


def _run_ref(rank):
    env = dict(os.environ, WORLD_SIZE="2", RANK=str(rank), LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--steps", "1", "--warmup", "3", "--rows", "256", "--ref-rows", "64"],
                          capture_output=True, text=True, env=env, timeout=300)


def test_reference_arm_rank0_prints_one_line_other_ranks_nothing():
    r1 = _run_ref(1)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _run_ref(0)
    assert r0.returncode == 0, r0.stderr
    lines = [ln for ln in r0.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == "GB/s" and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["cores"] == 1
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["e2e"]["d2h_bytes_per_step"] == 0
    assert rec["metric"] == bench.METRIC


def test_kernel_source_hash_ignores_comments_only():
    code = "int a;  // first\n/* a block\n   comment */ int b;\n\n  // only a comment\nint c;\n"
    assert bench._code_only(code) == "int a;\n int b;\nint c;"
    assert bench._code_only(code) == bench._code_only(code.replace("first", "changed"))
    assert bench._code_only(code) != bench._code_only(code.replace("int c;", "int c = 1;"))
    for k in bench.KERNEL_SOURCES:  # every listed source exists
        assert len(bench.sources_sha(k)) == 16


def test_recorded_traffic_only_for_matching_sources(tmp_path, monkeypatch):
    # a root with its own profiles/ and the real kernel sources
    os.symlink(os.path.join(bench.ROOT, "mxfp8_quantization_moe_mx_b200"),
               tmp_path / "mxfp8_quantization_moe_mx_b200")
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({
        "mx_dequantize": {"sources_sha": bench.sources_sha("mx_dequantize"), "dram_bytes_per_launch": 123},
        "per_group_quant": {"sources_sha": "0" * 16, "dram_bytes_per_launch": 456}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("mx_dequantize") == 123
    assert bench.recorded_traffic("per_group_quant") is None   # taken on other sources
    assert bench.recorded_traffic("mx_quantize_dual") is None  # never captured


def test_workload_names():
    assert bench.workload_name(bench.ROWS, bench.N_GROUPS) == bench.WORKLOAD
    assert "(16640, 5120)" in bench.workload_name(16640, 4) and "4 experts" in bench.workload_name(16640, 4)


def test_all_cores_oracle_step_equals_single_threaded():
    """The CPU baseline's slab split (row slabs for MX, column slabs for per-group, in
    spawned workers over shared memory) gives exactly the single-threaded oracle's
    step."""
    import numpy as np
    import oracle
    from oracle.parallel import StepOnAllCores
    from mxfp8_quantization_moe_mx_b200 import workloads as wl

    t = wl.dispatch(rows=640, cols=256, n_groups=5)
    xb = wl.bf16_bits(t["x"])
    offs = t["offs"].numpy()
    r = oracle.mx_quantize(xb, oracle.ROW | oracle.COL)
    y = oracle.mx_dequantize(r["q_row"], r["s_row"], 1, 640, 256, oracle.ROW)
    q, s = oracle.per_group_quant(y, offs, oracle.ROW_MAJOR)
    run = StepOnAllCores(xb, offs, workers=3)
    try:
        run.run()
        for k in ("q_row", "s_row", "q_col", "s_col"):
            np.testing.assert_array_equal(run.arr[k], r[k], err_msg=k)
        np.testing.assert_array_equal(run.arr["y"], y)
        np.testing.assert_array_equal(run.arr["q"], q)
        assert np.array_equal(run.arr["scales"].view(np.uint32), s.view(np.uint32))
    finally:
        run.close()


def test_cpu_baseline_record():
    """cpu_baseline: the all-cores figure with its core count, plus the single-threaded
    one, on a small batch."""
    import argparse
    from mxfp8_quantization_moe_mx_b200 import workloads as wl

    t = wl.dispatch(rows=256, cols=128, n_groups=4)
    rec = bench.cpu_baseline(t["x"], t["offs"], argparse.Namespace(cpu_rows=128))
    assert rec["kind"] == "oracle" and rec["unit"] == "GB/s" and rec["value"] > 0
    assert rec["cores"] >= 1 and rec["single_thread"]["cores"] == 1
    assert "256 x" not in rec["sample"] or "whole batch" in rec["sample"]


def test_clock_sampler_finds_the_gpu_by_pci_location(monkeypatch):
    """NVML numbers every GPU of the machine, CUDA only the visible ones: the sampler's
    handle is the NVML device at the CUDA device's PCI location, not NVML index 0."""
    from types import SimpleNamespace

    class FakeNvml:
        devices = [SimpleNamespace(domain=0, bus=0x18, device=0), SimpleNamespace(domain=0, bus=0x2A, device=0),
                   SimpleNamespace(domain=0, bus=0x9B, device=0)]

        def nvmlDeviceGetCount(self):
            return len(self.devices)

        def nvmlDeviceGetHandleByIndex(self, i):
            return ("handle", i)

        def nvmlDeviceGetPciInfo(self, h):
            return self.devices[h[1]]

    props = SimpleNamespace(pci_domain_id=0, pci_bus_id=0x9B, pci_device_id=0)
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda i: props)
    assert bench.nvml_handle(FakeNvml(), 0) == ("handle", 2)
    # no PCI match: the CUDA index is used as the NVML index
    props.pci_bus_id = 0x77
    assert bench.nvml_handle(FakeNvml(), 1) == ("handle", 1)


def test_clock_summary_uses_the_timed_region_then_the_steps_after_it():
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.max_mhz, s.errors, s.last_error, s._ok = 1965, 0, None, True
    s.samples = [(0.5, 1200), (1.1, 1965), (1.2, 1950), (1.3, 1965), (2.5, 1800)]
    s.masks = [(1.1, 0x4), (1.2, 0x1), (2.5, 0x20)]
    s.region(1.0, 1.4)
    r = s.summary()
    assert r["window"] == "timed region" and r["samples"] == 3 and r["sm_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]          # gpu_idle dropped, masks outside ignored
    # a region too short for three samples: the samples right after it are added
    s.region(1.0, 1.15)
    r = s.summary()
    assert r["samples"] == 4 and "after" in r["window"] and r["sm_mhz"] == 1957.5
    assert r["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"]
    # a failed read is reported, not hidden
    s.errors, s.last_error = 2, "NVMLError_NotSupported"
    assert s.summary()["nvml_errors"] == 2
