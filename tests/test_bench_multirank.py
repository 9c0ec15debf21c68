"""The benchmark's multi-rank path on CPU: two gloo ranks (one process each,
127.0.0.1 rendezvous) take the max of their times and report the whole-job
throughput, as bench.py does with NCCL on GPUs."""
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
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + rank, 20.0 - rank]          # rank 1 is slower on the first value
        got = bench.max_over_ranks(mine, dist, torch.device("cpu"))
        value = bench.whole_job_tflops(world, 1e12, got[0])
        dist.barrier()
        q.put((rank, got, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_whole_job_value():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    out = sorted(q.get(timeout=10) for _ in range(world))
    for rank, got, value in out:
        assert got == [11.0, 20.0]                 # max over ranks, element by element
        assert value == pytest.approx(2 * 1e12 / 11e-3 / 1e12)


def test_single_rank_is_identity():
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    assert bench.whole_job_tflops(1, 2e12, 1000.0) == pytest.approx(2.0)
