"""The N > 1 path of bench.py on CPU: two gloo ranks (replicas, no collective
on the data path) agree on the slowest rank's time and on the whole-job rate."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        local_ms = [30.0, 45.5][rank]                   # rank 1 is slower
        total = bench.max_over_ranks(local_ms, torch.device("cpu"))
        rate = bench.whole_job_rate(1e9, world, 10, total)
        results[rank] = (total, rate)
    finally:
        dist.destroy_process_group()


def test_two_replicas_report_the_slowest_rank():
    port = _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_rank, args=(2, port, results), nprocs=2, join=True, start_method="spawn")
        got = dict(results)
    assert got[0] == got[1]
    total, rate = got[0]
    assert total == 45.5
    assert rate == pytest.approx(1e9 * 2 * 10 / 45.5e-3)


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(12.5, torch.device("cpu")) == 12.5
    assert bench.whole_job_rate(4.0, 1, 5, 1000.0) == pytest.approx(20.0)
