"""The benchmark's multi-process plumbing on CPU: two gloo ranks.

bench.py runs one independent replica of the workload per GPU (the path has
no exchange step), so the only collectives are the barrier around the timed
region and the max over ranks of the measured time.  These run here with the
gloo backend, world size 2, no GPU.
"""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def worker(rank, world, port, results):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w, r, lr = bench.dist_init(world)
        bench.barrier(world)
        # each rank timed a different duration; every rank must report the max
        t = bench.max_over_ranks(10.0 * (rank + 1), world, torch.device("cpu"))
        results[rank] = (w, r, lr, t)
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_over_ranks_and_barrier():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = free_port()
        procs = [ctx.Process(target=worker, args=(r, 2, port, results)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        assert dict(results) == {0: (2, 0, 0, 20.0), 1: (2, 1, 1, 20.0)}


def test_single_process_needs_no_collective():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    bench.barrier(1)


def test_world_size_mismatch_is_rejected(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "4")
    with pytest.raises(SystemExit):
        bench.dist_init(2)
