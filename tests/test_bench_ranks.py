"""Multi-rank host logic of bench.py on CPU: two gloo ranks (one process per
rank, as torchrun starts them) check the max-over-ranks timing, the whole-job
rate, the per-rank seeds and that only rank 0 runs and prints the oracle arm.
The decode path itself shards by sequence and has no collective."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, results):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms = [3.5, 7.25][rank]                       # per-rank device times
        got = bench.max_over_ranks(ms, world, "cpu")
        rate = bench.whole_job_rate(1000, world, 10, got)
        seeds = [bench.layer_seed(rank, l) for l in range(8)]
        gathered = [None] * world
        dist.all_gather_object(gathered, seeds)
        out = io.StringIO()
        if rank != 0:
            class Args:
                steps, warmup, layers = 2, 3, 8
            with redirect_stdout(out):
                bench.reference_arm(Args, bench.WORKLOADS["qwen35_9b_gdn"], rank, world)
        dist.barrier()
        results[rank] = (got, rate, gathered, out.getvalue())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), results), nprocs=world,
                           join=True, start_method="spawn")
        res = dict(results)
    assert sorted(res) == [0, 1]
    for rank in range(world):
        got, rate, gathered, printed = res[rank]
        assert got == 7.25                             # the slowest rank's time
        assert rate == pytest.approx(2 * 1000 * 10 / 7.25e-3)
        flat = [s for seeds in gathered for s in seeds]
        assert len(set(flat)) == len(flat)             # no two ranks share a layer's data
    assert res[1][3] == ""                             # rank 1 prints nothing


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert not dist.is_initialized()
    assert bench.max_over_ranks(4.0, 1) == 4.0
    assert bench.whole_job_rate(5, 1, 2, 1000.0) == pytest.approx(10.0)


def test_reference_arm_line_keeps_the_contract(monkeypatch):
    """Rank 0 of --impl reference prints one JSON line with the contract's keys:
    the oracle timed on host cores, its own e2e with no transfers."""
    sys.path.insert(0, ROOT)
    import bench

    monkeypatch.setattr(bench, "REFERENCE_BUDGET_S", 0.6)

    class Args:
        steps, warmup, layers = 2, 1, 8

    out = io.StringIO()
    with redirect_stdout(out):
        bench.reference_arm(Args, bench.WORKLOADS["qwen35_9b_gdn"], 0, 1)
    lines = out.getvalue().strip().splitlines()
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["unit"] == bench.UNIT and d["metric"] == bench.METRIC
    assert d["value"] > 0 and d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["higher_is_better"] is True and d["vs_baseline"] is None
    assert d["config"]["workload"] == bench.WORKLOADS["qwen35_9b_gdn"].name
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_clock_sampler_summary_parses_nvidia_smi_lines():
    """The clocks object of the bench line: median SM clock under load, the max
    clock, and the throttle reasons seen inside the timed window only."""
    sys.path.insert(0, ROOT)
    import bench

    cs = bench.ClockSampler(None)
    na = "Not Active"
    cs.lines = [
        (0.5, f"1200, 1965, 300.0, 0x0, {na}, {na}, {na}, {na}"),        # before the window
        (1.0, f"1965, 1965, 700.0, 0x0, {na}, {na}, {na}, {na}"),
        (1.1, f"1950, 1965, 990.0, 0x4, {na}, {na}, {na}, Active"),      # power cap
        (1.2, f"1965, 1965, 800.0, 0x0, {na}, {na}, {na}, {na}"),
        (1.3, "garbled"),                                                 # skipped
        (3.0, f"900, 1965, 200.0, 0x8, Active, {na}, {na}, {na}"),       # after the window
    ]
    cs.window(0.9, 1.5)
    s = cs.summary()
    assert s == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                 "samples": 3}
    cs.window(0.0, 10.0)
    s = cs.summary()
    assert s["reasons"] == ["hw_slowdown", "sw_power_cap"] and s["samples"] == 5
    empty = bench.ClockSampler(None)
    assert empty.summary()["reasons"] == ["no samples"]


def test_algorithmic_bytes_and_profiled_traffic(tmp_path, monkeypatch):
    """The roofline's numerator: bytes one tile-step must move, item by item
    (record from the public layout, a half-full window's buffer on average,
    shared keys split over the value heads of a key head); and the DRAM
    traffic read from the ncu summary only while the kernel source matches
    the hash it was captured on."""
    sys.path.insert(0, ROOT)
    import bench

    w = bench.WORKLOADS["qwen35_9b_gdn"]
    ab = bench.algorithmic_bytes_per_tile_step(w)
    d, g = 128, 2
    record = d * d + 4 * d + 4 * d + 4 * 4 * d + 4 * 4          # codes, sigma, m, lines, ids
    entry = 4 * d + 4 + 2 * d / g                               # d_s, alpha_s, half a bf16 k_s
    assert ab == {"record_read": record, "buffer_read": 7.5 * entry, "buffer_append": entry,
                  "fold_record_write": record / 16, "inputs": 2 * 2 * d / g + 2 * d + 8,
                  "output": 4 * d, "phase_counter": 8, "total": 27203.0}
    assert record == 19472
    assert bench.fp32_bytes_per_tile_step(w) == 2 * 4 * d * d + 520 + 4 * d

    src = tmp_path / "kernel.cu"
    src.write_text("// kernel\nint v = 1;\n")
    monkeypatch.setattr(bench, "KERNEL_SOURCES", [str(src)])
    summary = tmp_path / "decode_kernel_qwen35_9b_gdn.md"
    monkeypatch.setattr(bench, "PROFILE_DIR", str(tmp_path))
    assert bench.profile_summary_path("qwen35_9b_gdn") == str(summary)
    assert bench.profiled_traffic(10) is None                   # no summary
    summary.write_text(f"kernel_source_sha: {bench.kernel_source_sha()}\n"
                       "dram_bytes_per_tile_step: 24911\n")
    assert bench.profiled_traffic(2048) == 24911 * 2048
    assert bench.profiled_traffic(4096, "kimi_linear_kda") is None   # another workload's file
    src.write_text("/* the kernel,\n   reworded */ int v = 1;  // same code\n")
    assert bench.profiled_traffic(2048) == 24911 * 2048        # comments alone changed
    src.write_text("// kernel\nint v = 2;\n")                  # kernel changed since
    assert bench.profiled_traffic(2048) is None
    # the roofline names the kernel instance of each workload
    assert bench.kernel_label(bench.WORKLOADS["kimi_linear_kda"]).startswith(
        "decode_kernel<128,bf16,KDA>")
    assert bench.kernel_label(w).startswith("decode_kernel<128,bf16,GDN>")


def test_working_set_and_l2_statement():
    """The config's L2 statement: the step's working set (every layer's state
    per the C library's layout, its W tokens of inputs and its output) decides
    whether a run streams from HBM or sits in the 126 MB L2."""
    sys.path.insert(0, ROOT)
    import bench
    from recurrent_state_quantization_decode_b200 import binding as B

    for name in ("qwen35_9b_gdn", "kimi_linear_kda", "gdn_sweep_b8"):
        w = bench.WORKLOADS[name]
        L = B.lq_state_layout(B.config_for(w))
        state = (L.records_bytes + L.buf_k_bytes + L.buf_d_bytes + L.buf_g_bytes
                 + L.buf_n_bytes)
        inb = 2 if w.io_bf16 else 4
        ga = w.d if w.gate == 1 else 1
        inputs = w.window * (2 * w.batch * w.num_k_heads * w.d * inb
                             + w.tiles * w.d * inb + w.tiles * ga * 4 + w.tiles * 4)
        out = w.tiles * w.d * 4
        assert bench.working_set_bytes(w, 8) == 8 * (state + inputs + out), name
    big = bench.workload_config(bench.WORKLOADS["qwen35_9b_gdn"], 8)
    assert big["l2"].startswith("inputs larger than L2") and big["working_set_mb"] > 2 * 126
    small = bench.workload_config(bench.WORKLOADS["gdn_sweep_b8"], 8)
    assert "L2-resident" in small["l2"] and small["working_set_mb"] < 126
