"""Host logic of the user-sharded replica serving, on CPU: the owner hash,
the slot table, and two gloo ranks that split a batch of users without
overlap and gather their per-user scores on rank 0."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from unified_transformer_recommender_b200 import serving


def test_owner_rank_covers_every_rank_evenly():
    for world in (1, 2, 3, 8):
        counts = [0] * world
        for u in range(20000):
            r = serving.owner_rank(u, world)
            assert 0 <= r < world
            counts[r] += 1
        assert min(counts) >= 0.9 * 20000 / world, counts
    assert serving.owner_rank(12345, 8) == serving.owner_rank(12345, 8)
    parts = serving.route([7, 3, 7 + 2 ** 40, 11], 2)
    assert sorted(i for v in parts.values() for i in v) == [0, 1, 2, 3]


def test_slot_table_keeps_evicts_least_recently_used():
    t = serving.SlotTable(3)
    assert t.assign([10, 11, 12]) == [0, 1, 2]
    assert t.assign([11]) == [1]                # present: keeps its slot
    assert t.lookup([10]) == [0]                # 12 is now the least recently used
    assert t.assign([13]) == [2] and 12 not in t
    with pytest.raises(KeyError):
        t.lookup([12])
    assert t.assign([14, 10]) == [1, 0]         # 11 evicted, never a user of this batch
    assert 11 not in t and 13 in t
    with pytest.raises(ValueError):
        t.assign([1, 1])
    with pytest.raises(ValueError):
        t.assign([1, 2, 3, 4])
    t.evict(13)
    assert t.assign([15]) == [2]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    users = list(range(64))
    mine = [u for u in users if serving.owner_rank(u, world) == rank]
    scores = torch.tensor([[1.5 * u, -u] for u in mine], dtype=torch.float32).reshape(len(mine), 2)
    got = serving.gather_to_rank0(mine, scores)
    q.put((rank, mine, None if got is None else {u: v.tolist() for u, v in got.items()}))
    dist.destroy_process_group()


def test_two_ranks_split_users_and_gather_scores_on_rank0():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, mine0, got0), (_, mine1, got1) = res
    assert sorted(mine0 + mine1) == list(range(64)) and not set(mine0) & set(mine1)
    assert got1 is None and sorted(got0) == list(range(64))
    assert all(got0[u] == [1.5 * u, -u] for u in range(64))
