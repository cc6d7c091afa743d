"""The benchmark's multi-GPU host logic on CPU: two gloo ranks shard users
without overlap and agree on the max-over-ranks device time."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    users = bench.shard_users(16, rank)
    got = [None] * world
    dist.all_gather_object(got, users)
    t = bench.max_over_ranks(10.0 + 5.0 * rank)
    q.put((rank, got, t, bench.dist_env()))
    dist.destroy_process_group()


def test_two_rank_user_sharding_and_max_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, t, env in res:
        flat = [u for part in got for u in part]
        assert sorted(flat) == list(range(32)) and len(set(flat)) == 32
        assert t == 15.0
        assert env == (2, rank, 0)
