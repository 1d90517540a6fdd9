"""The multi-process plumbing of bench.py on CPU: two gloo ranks, as torchrun
would start them on two GPUs. Each rank runs its own copy of the workload (no
data exchange); the job's step time is the slowest rank's, and the reported
rate counts the units of every rank."""
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


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms_local = 2.0 + rank            # rank 1 is the slower one
        ms = bench.reduce_max(ms_local, world)
        rate = bench.aggregate_rate(4096, ms, world)
        results[rank] = (ms, rate)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank_and_sum_the_work():
    world, port = 2, _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, results), nprocs=world, join=True)
        got = dict(results)
    assert set(got) == {0, 1}
    for ms, rate in got.values():
        assert ms == pytest.approx(3.0)
        assert rate == pytest.approx(2 * 4096 / 3e-3)


def test_single_rank_needs_no_process_group():
    assert bench.reduce_max(1.25, 1) == 1.25
    assert bench.aggregate_rate(10, 2.0, 1) == pytest.approx(5000.0)
