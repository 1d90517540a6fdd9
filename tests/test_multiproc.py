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


def test_reference_arm_as_two_ranks_prints_one_line_from_rank_0():
    """`bench.py --impl reference` launched as two ranks the way a multi-GPU run is
    launched: rank 0 alone times the oracle on the host cores and prints one JSON
    line; the other rank exits 0 without work. No GPU or process group is needed."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}", "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["dtype"] == "f64"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
