"""The N > 1 host logic of bench.py on CPU: two gloo ranks, max-over-ranks timing, weak scaling.

Each rank runs its own batch (the loss shards by tokens with no exchange), so the only
cross-rank steps are the barrier and the max of the step times; these run here without a GPU.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys

    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        local = [1.5, 2.5][rank]  # seconds this rank took for its steps
        slowest = bench.max_over_ranks(local, world, torch.device("cpu"))
        value = bench.weak_scaling_value(world, 4096, 10, slowest)
        out[rank] = (slowest, value)
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:  # no fork of this multi-threaded process
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    assert res[0] == res[1]
    slowest, value = res[0]
    assert slowest == 2.5
    assert value == pytest.approx(2 * 4096 * 10 / 2.5)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import sys

    sys.path.insert(0, ROOT)
    import bench

    class Args:
        workload, steps, warmup, ref_rows, gpus = "tiny", 1, 0, 8, 2

    bench.run_reference(Args, world=2, rank=1)  # a non-zero rank does no work and prints nothing
    assert capsys.readouterr().out == ""


def test_issued_backward_work():
    """The backward's issued tensor-core work: recompute and dE over kept 128 x 64 units, dC over
    both units of every 128 x 128 tile with a kept unit."""
    import torch
    import bench

    # 2 row blocks x 5 units (the last tile has one unit): 0 = kept, 1 = skipped
    skip_map = torch.tensor([[0, 1, 1, 1, 1],
                             [1, 0, 0, 0, 0]], dtype=torch.uint8)
    assert bench.listed_tile_count(skip_map) == 1 + 3
    kept_units = int((skip_map == 0).sum())
    assert kept_units == 5
    D = 256
    assert bench.issued_mma_flops(D, kept_units, 4, (128, 64)) == \
        4 * 128 * 64 * D * 5 + 2 * 128 * 128 * D * 4


def test_algorithmic_flops_definition():
    """The metric's flop count: 2 N V D forward, 6 * 128 * 64 * D per kept 128 x 64 unit of the skip
    rule (recompute, dE and dC of its logits)."""
    import bench

    fwd, bwd = bench.algorithmic_flops(4096, 4096, 128256, 8062, (128, 64))
    assert fwd == 2 * 4096 * 128256 * 4096
    assert bwd == 6 * 128 * 64 * 4096 * 8062
    # every workload of the bench has N and V multiples of 128 (no partial unit is counted)
    from linear_cross_entropy_06_b200.inputs import WORKLOADS
    for w in WORKLOADS.values():
        if w.name != "tiny":
            assert w.N % 128 == 0 and w.V % 128 == 0, w.name


def test_reference_arm_prints_the_contract_line(capsys, monkeypatch):
    """--impl reference on rank 0: one JSON line timing the fp64 oracle on the host, with its own
    cpu_baseline and an e2e that moves no bytes; the CUDA library is never loaded for it."""
    import json
    import sys

    sys.path.insert(0, ROOT)
    import bench
    from linear_cross_entropy_06_b200 import ops

    def refuse(*a, **k):
        raise AssertionError("the reference arm loaded the CUDA library")

    monkeypatch.setattr(ops, "load_library", refuse)

    class Args:
        workload, steps, warmup, ref_rows, gpus = "tiny", 2, 1, 16, 1

    bench.run_reference(Args, world=1, rank=0)
    out = capsys.readouterr().out.strip().splitlines()
    assert len(out) == 1
    line = json.loads(out[0])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True and line["value"] > 0
    assert line["steps"] == 2 and line["warmup"] == 1 and line["n_gpus"] == 1
    assert line["config"]["workload"] == "tiny"
    cpu = line["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["value"] == line["value"] and cpu["cores"] >= 1 and cpu["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert bench.ORACLE_SKIP_TILE == (128, 64)
    # cores = the BLAS pool that runs the oracle's matmul, at least one thread and at most the host's CPUs
    assert cpu["cores"] == bench.oracle_threads() and 1 <= cpu["cores"] <= (os.cpu_count() or 1)


def test_clock_sampler_parses_samples_and_reasons(monkeypatch):
    """The clocks object of the bench line, from nvidia-smi's CSV: median SM clock under load (idle
    samples below half the top clock are left out), max clock, and every throttle reason seen."""
    import subprocess
    import sys

    sys.path.insert(0, ROOT)
    import bench

    samples = [
        "0, 345, 1965, 120.5, 0x0, Not Active, Not Active, Not Active, Not Active, 1000.00",
        "0, 1965, 1965, 650.0, 0x4, Not Active, Not Active, Not Active, Active, 1000.00",
        "0, 1950, 1965, 700.2, 0x4, Not Active, Not Active, Not Active, Active, 1000.00",
        "0, 1905, 1965, 710.9, 0x0, Not Active, Not Active, Not Active, Not Active, 1000.00",
    ]

    class FakeSmi:
        def __init__(self, cmd, stdout=None, stderr=None):
            assert cmd[0] == "nvidia-smi" and "-lms" in cmd
            stdout.write("\n".join(samples) + "\n")
            stdout.flush()

        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    monkeypatch.setattr(subprocess, "Popen", FakeSmi)
    monkeypatch.setattr(bench.time, "sleep", lambda s: None)
    c = bench.ClockSampler(0)
    c.start()
    out = c.stop()
    assert out["sm_mhz"] == 1950.0  # median of 1965, 1950, 1905; the idle 345 is left out
    assert out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]
    assert out["samples"] == 4 and out["power_w_max"] == 710.9 and out["power_limit_w"] == 1000.0
    assert not os.path.exists(c.path)


def test_roofline_traffic_is_dropped_when_the_kernel_changes(monkeypatch):
    """The roofline's DRAM traffic is a past ncu capture; it is reported only while the kernel's
    sources hash to the value recorded with it, and is null for any other shape."""
    import sys

    sys.path.insert(0, ROOT)
    import bench

    sha = bench.kernel_source_hash("bwd_kernel")
    assert len(sha) == 64 and sha == bench.kernel_source_hash("bwd_kernel")
    assert sha != bench.kernel_source_hash("fwd_lse_kernel")
    monkeypatch.setitem(bench.TRAFFIC_BYTES, "bwd_kernel", {(4096, 4096, 128256): (sha, 123456789)})
    assert bench.measured_traffic("bwd_kernel", (4096, 4096, 128256)) == 123456789
    assert bench.measured_traffic("bwd_kernel", (2048, 2048, 128256)) is None
    monkeypatch.setitem(bench.TRAFFIC_BYTES, "bwd_kernel", {(4096, 4096, 128256): ("0" * 64, 123456789)})
    assert bench.measured_traffic("bwd_kernel", (4096, 4096, 128256)) is None
