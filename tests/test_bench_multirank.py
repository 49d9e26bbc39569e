"""The N > 1 host path of bench.py on CPU, with world-size-2 gloo process groups.

bench.py runs replicas (every rank its own full step on its own batch, no data-path
collective); the only cross-rank step is the timing reduction: the job takes the slowest rank's
device time, and the whole-job throughput counts every rank's batch. The reference arm runs on
rank 0 alone.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slower one
        job_ms = bench.max_over_ranks(local_ms, world, dist, "cpu")
        # a second reduction in the same order on every rank (the bench reduces twice)
        job_ms2 = bench.max_over_ranks(2.0 * local_ms, world, dist, "cpu")
        out[rank] = (job_ms, job_ms2)
    finally:
        dist.destroy_process_group()


def test_timing_is_the_max_over_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert res == {0: (15.0, 30.0), 1: (15.0, 30.0)}


def test_whole_job_throughput_counts_every_replica():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.whole_job_tflops(1, 5.37e12, 2.5)
    assert abs(one - 5.37e12 / 2.5e-3 / 1e12) < 1e-9
    assert abs(bench.whole_job_tflops(4, 5.37e12, 2.5) - 4 * one) < 1e-9
    assert bench.max_over_ranks(3.5, 1, None, "cpu") == 3.5  # one rank: no collective at all


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.run_reference(type("A", (), {"workload": "ffn5b", "cpu_rows": 2, "warmup": 1, "steps": 1})())
    assert capsys.readouterr().out == ""
