"""Multi-rank host logic on the CPU (gloo, world size 2): request sharding, the
max-over-ranks timing reduction, the aggregate rate, and a rank that dies before a
collective (the survivor gets an error instead of waiting for ever)."""

import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from masked_block_diffusion_b200.replicas import aggregate_rate, max_over_ranks, shard_requests


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _init(rank, world, port, timeout_s=30):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=timeout_s))


def _worker_timing(rank, world, port, q):
    _init(rank, world, port)
    mine = shard_requests(64, world, rank)
    t = [0.5, 1.25][rank]                     # per-rank "elapsed seconds"
    dist.barrier()
    m = max_over_ranks(t, "cpu")
    q.put((rank, mine, m))
    dist.barrier()
    dist.destroy_process_group()


def _worker_dies(rank, world, port, q):
    _init(rank, world, port, timeout_s=5)
    if rank == 1:
        os._exit(3)                            # leaves between steps, before the collective
    try:
        dist.barrier()
        q.put((rank, "no error"))
    except Exception as e:                     # timeout / connection closed
        q.put((rank, type(e).__name__))


def test_shard_requests_cover_disjoint():
    for n, w in ((64, 8), (5, 2), (1, 4), (0, 3)):
        parts = [shard_requests(n, w, r) for r in range(w)]
        flat = sorted(i for p in parts for i in p)
        assert flat == list(range(n))
    with pytest.raises(ValueError):
        shard_requests(4, 2, 2)


def test_aggregate_rate():
    assert aggregate_rate(256, 4, 2.0) == 512.0
    with pytest.raises(ValueError):
        aggregate_rate(1, 1, 0.0)


def test_two_rank_timing_reduction():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker_timing, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(2))
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, mine0, m0), (r1, mine1, m1) = out
    assert m0 == m1 == 1.25
    assert sorted(mine0 + mine1) == list(range(64)) and not set(mine0) & set(mine1)


def test_dead_rank_is_detected_by_the_survivor():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker_dies, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    rank, what = q.get(timeout=120)
    for p in ps:
        p.join(timeout=60)
    assert rank == 0 and what != "no error"
    assert ps[1].exitcode == 3
