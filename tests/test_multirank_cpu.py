"""The N > 1 path of bench.py on the CPU with gloo, world size 2.

The path shards by independent problems (every (b, d) channel is its own
recurrence), so the only cross-rank traffic is the timing reduction: each rank
times its own problem, the job time is the max over ranks, and the job value
counts every rank's elements.  Ranks draw different seeds."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), LOCAL_RANK=str(rank),
                      WORLD_SIZE=str(world))
    import bench
    import torch

    r, lr, w = bench.dist_env()
    dist = bench.dist_init("gloo", w)
    try:
        bench.barrier(dist)
        my_ms = 10.0 + 5.0 * rank  # rank 1 is the slower one
        mx = bench.reduce_max(dist, my_ms, torch.device("cpu"))
        seeds = [None] * w
        dist.all_gather_object(seeds, bench.rank_seed(4, r))
        q.put((r, lr, w, mx, seeds, bench.aggregate_throughput(1000, w, 3, mx)))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_ranks_time_is_max_and_value_counts_all_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=90) for _ in range(world))
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for r, (rank, lr, w, mx, seeds, value) in enumerate(res):
        assert rank == r and lr == r and w == world
        assert mx == 15.0  # the slowest rank's time
        assert len(set(seeds)) == world  # independent problems
        assert value == pytest.approx(1000 * world * 3 / 0.015)


def test_single_process_defaults(monkeypatch):
    import bench

    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_env() == (0, 0, 1)
    assert bench.dist_init("gloo", 1) is None
    assert bench.reduce_max(None, 3.5, None) == 3.5
