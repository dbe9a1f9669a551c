"""The multi-rank plumbing of bench.py on CPU: two gloo ranks take the same
collective steps, the timing is the max over ranks and the whole-job
throughput counts every rank's work (weak scaling: one replica per rank)."""
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, init_method=f"tcp://127.0.0.1:{port}")
    try:
        dist.barrier()
        # rank r pretends its step took (r + 1) ms and its Stage 2 (10 - r) ms
        got = bench.max_over_ranks([rank + 1.0, 10.0 - rank], world, torch.device("cpu"))
        dist.barrier()
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_throughput():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == res[1] == [2.0, 10.0]
    # whole-job value: every rank's work over the slowest rank's time
    assert bench.job_throughput(1e12, world, 2.0) == pytest.approx(1e15)


def test_single_rank_is_identity():
    assert bench.max_over_ranks([3.0, 4.0], 1, torch.device("cpu")) == [3.0, 4.0]
