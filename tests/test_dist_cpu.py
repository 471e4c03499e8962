"""The multi-rank host logic of bench.py on CPU: world size 2 over gloo.

Each rank runs an independent stream (its own seed); the job's time is the max over ranks of
the per-rank device time.  No collective touches the layer's data."""
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
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, lr, w = bench.dist_env()
        assert (r, lr, w) == (rank, rank, world)
        t = bench.reduce_max(1.5 + rank, w)                 # ranks report 1.5 and 2.5 ms
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.rank_seed(2024, rank))
        q.put((rank, t, seeds))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_max_time_and_distinct_streams():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [t for _, t, _ in res] == [2.5, 2.5]
    seeds = res[0][2]
    assert len(set(seeds)) == 2


def test_single_rank_defaults(monkeypatch):
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_env() == (0, 0, 1)
    assert bench.reduce_max(3.0, 1) == 3.0
