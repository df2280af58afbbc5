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
    with mp.Manager() as m:
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


def test_algorithmic_flops_definition():
    """The metric's flop count: 2 N V D forward, 6 * 128 * 128 * D per kept 128 x 128 tile."""
    import bench

    fwd, bwd = bench.algorithmic_flops(4096, 4096, 128256, 7407, (128, 128))
    assert fwd == 2 * 4096 * 128256 * 4096
    assert bwd == 6 * 128 * 128 * 4096 * 7407
    # every workload of the bench has N and V multiples of 128 (no partial tile is counted)
    from linear_cross_entropy_06_b200.inputs import WORKLOADS
    for w in WORKLOADS.values():
        if w.name != "tiny":
            assert w.N % 128 == 0 and w.V % 128 == 0, w.name
