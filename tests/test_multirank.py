"""The multi-rank logic of bench.py with two gloo ranks on the CPU: the device
time is the max over ranks, the value counts the work of every rank, and the
reference arm runs on rank 0 only. CPU only."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 100.0 + 50.0 * rank            # rank 1 is the slow one
        total = bench.max_over_ranks(local_ms, world, "cpu")
        value = bench.job_throughput(32768, world, 10, total)
        dist.barrier()

        class A:   # the reference arm's arguments
            workload, steps, warmup, gpus, ref_tokens = 3, 1, 0, world, 4
        if rank != 0:
            bench.run_reference(A, rank)           # returns at once, no work, no output
        q.put((rank, total, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_count_all_work():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, total, value in res:
        assert total == 150.0                       # the slowest rank's time
        assert value == pytest.approx(2 * 32768 * 10 / 0.150)


def test_single_rank_is_the_identity():
    assert bench.max_over_ranks(12.5, 1, "cpu") == 12.5
    assert bench.job_throughput(100, 1, 4, 200.0) == pytest.approx(2000.0)
