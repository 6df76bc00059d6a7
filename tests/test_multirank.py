"""The multi-rank logic of bench.py with two gloo ranks on the CPU: the device
time is the max over ranks, the value counts the work of every rank, and the
reference arm runs on rank 0 only; the ranks' head shares cover every (b,
kv-head) unit once. CPU only."""
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


@pytest.mark.parametrize("B,Hkv,world", [(1, 8, 1), (1, 8, 2), (1, 8, 4), (1, 8, 8), (16, 8, 4),
                                         (2, 8, 4), (1, 6, 4)])
def test_head_shards_cover_every_unit_once(B, Hkv, world):
    # the ranks' shares of the (b, kv-head) units are contiguous, disjoint, cover all
    # units and differ in size by at most one
    shards = [bench.head_shard(B, Hkv, world, r) for r in range(world)]
    assert shards[0][0] == 0 and shards[-1][1] == B * Hkv
    assert all(shards[r][1] == shards[r + 1][0] for r in range(world - 1))
    sizes = [u1 - u0 for u0, u1 in shards]
    assert max(sizes) - min(sizes) <= 1


def test_head_shard_data_equals_the_full_draw():
    # a rank draws only its kv-heads (with their query heads) and gets exactly the
    # slices of the full workload
    from workloads import PARITY_WORKLOADS, generate
    w = PARITY_WORKLOADS["p_bf16_blk128"].with_(B=1)
    full = generate(w)
    G = w.Hq // w.Hkv
    for r in range(2):
        g0, g1 = bench.head_shard(1, w.Hkv, 2, r)
        part = generate(w, heads=[(0, g) for g in range(g0, g1)])
        assert (part["q"][:, g0 * G:g1 * G] == full["q"][:, g0 * G:g1 * G]).all()
        assert (part["k"][:, g0:g1] == full["k"][:, g0:g1]).all()
        assert (part["v"][:, g0:g1] == full["v"][:, g0:g1]).all()
