"""Multi-rank plumbing of bench.py, on CPU with two gloo ranks: the slowest
rank's time is what every rank reports, the whole-job throughput counts the
units of all ranks over that time, replicas draw distinct data, and the
reference arm does its work on rank 0 only."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as tmp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank            # rank 1 is the slow one
        m = bench.max_over_ranks(local_ms, world, "cpu")
        results[rank] = (m, bench.job_throughput(16 * 64, world, m), bench.rank_seed_offset(rank))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world = 2
    with tmp.Manager() as mgr:
        results = mgr.dict()
        tmp.spawn(_worker, args=(world, _free_port(), results), nprocs=world, join=True)
        res = dict(results)
    assert res[0][0] == res[1][0] == 15.0
    assert res[0][1] == pytest.approx(2 * 16 * 64 / 15e-3)
    assert res[0][2] != res[1][2]


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.job_throughput(100, 1, 2.0) == pytest.approx(50000.0)


def test_reference_arm_runs_on_rank0_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        steps, warmup = 1, 3
    assert bench.run_reference(A()) == 0
    assert capsys.readouterr().out == ""


def test_decode_traffic_is_reported_only_for_the_profiled_sources(monkeypatch):
    import bench
    assert bench.decode_traffic() in (None, bench.DECODE_TRAFFIC["bytes_per_launch"])
    monkeypatch.setitem(bench.DECODE_TRAFFIC, "sha256", "0" * 64)
    assert bench.decode_traffic() is None
