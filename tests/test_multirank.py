"""Multi-rank host logic of bench.py on CPU: two gloo ranks (spawned processes).

The path has no exchange step, so N GPUs run N replicas; the job's throughput is
every rank's tokens over the slowest rank's device time, and only rank 0 runs the
CPU reference arm.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [10.0, 25.0][rank]            # rank 1 is the slow replica
        value, ms_step = bench.replica_throughput(16384, local_ms, 5, world)
        bench.barrier(world)
        out[rank] = (value, ms_step)
    finally:
        dist.destroy_process_group()


def test_replica_throughput_two_gloo_ranks():
    world = 2
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    # both ranks see the slowest rank's time: 25 ms / 5 steps = 5 ms per step
    for r in range(world):
        value, ms_step = out[r]
        assert ms_step == pytest.approx(5.0)
        assert value == pytest.approx(2 * 16384 / 5e-3)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        steps, warmup, gpus = 1, 3, 2

    # rank 1 returns at once, without building or running the oracle
    assert bench.run_reference(A()) == 0


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    value, ms_step = bench.replica_throughput(1000, 40.0, 4, 1)
    assert ms_step == pytest.approx(10.0)
    assert value == pytest.approx(1000 / 10e-3)


def test_clock_summary_window_and_reasons():
    """The clock record keeps only samples inside the timed window: median SM clock, the
    highest max clock, and the union of the active reasons."""
    sys.path.insert(0, ROOT)
    import bench
    cs = bench.ClockSampler(0)
    cs.source = "test"
    cs.samples = [(0.5, 900.0, 1965.0, {"hw_slowdown"}),          # before the window
                  (1.0, 1950.0, 1965.0, set()),
                  (1.1, 1900.0, 1965.0, {"sw_power_cap"}),
                  (1.2, 1935.0, 1965.0, set()),
                  (3.0, 600.0, 1965.0, {"sw_thermal_slowdown"})]   # after it
    got = cs.summary(1.0, 2.0)
    assert got == {"sm_mhz": 1935.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3,
                   "source": "test"}
    assert cs.summary(5.0, 6.0) is None
