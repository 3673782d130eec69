"""The multi-GPU host logic of bench.py on CPU with two gloo ranks: the path
needs no collective ("replicas only"), each rank draws its own batch, the time
is the max over ranks and the value counts every rank's tokens."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
    got = bench.max_over_ranks(ms, dist, "cpu")
    seeds = [bench.rank_seed(1001, rank, world, i) for i in range(3)]
    q.put((rank, got, seeds))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_distinct_batches():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(got == 15.0 for _, got, _ in out)  # every rank sees the slowest rank's time
    seeds = [s for _, _, ss in out for s in ss]
    assert len(set(seeds)) == len(seeds)  # no two (rank, replica) share a batch


def test_whole_job_rate_counts_all_ranks():
    import bench
    assert bench.whole_job_rate(4096, 20, 8, 100.0) == pytest.approx(4096 * 20 * 8 / 0.1)
    assert bench.max_over_ranks(3.0, None, "cpu") == 3.0
