"""User-sharded replica serving: one process per GPU, each a full replica of
the model holding the KV cache of the users it owns.

Stage I, Stage II and the cross-request append of one user touch only that
user's cached S-side keys and values and the shared weights ([FR] 7.5.3, the
two-stage cache; paper-daily 6.3, cross-request KV cache in serving), so
users are partitioned across GPUs with no collective on the data path: a
request goes to the rank that owns its user, and scores travel back to a
front end only if the caller asks (`gather_to_rank0`).

Host bookkeeping only: every step of the path runs in the library's kernels
through the C ABI.  The owner of a user is a fixed hash of its id, so every
process computes it without communication; a rank keeps its users in the
slots of one cache and evicts the least recently used user when a new one
needs a slot.
"""
from __future__ import annotations

import collections
from typing import Dict, List, Optional, Sequence

import torch

from . import (OP_APPEND, OP_STAGE1, OP_STAGE2, Cache, Model, onetrans_cache_append, onetrans_stage1_encode,
               onetrans_stage2_score)

_M64 = (1 << 64) - 1


def owner_rank(user_id: int, world: int) -> int:
    """The rank that serves `user_id`: splitmix64(user_id) mod world."""
    z = (int(user_id) + 0x9E3779B97F4A7C15) & _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    z ^= z >> 31
    return z % world


def route(user_ids: Sequence[int], world: int) -> Dict[int, List[int]]:
    """Positions of a request batch's users per owning rank (ranks without
    users omitted), in the batch's order."""
    out: Dict[int, List[int]] = collections.defaultdict(list)
    for i, u in enumerate(user_ids):
        out[owner_rank(u, world)].append(i)
    return dict(out)


class SlotTable:
    """User id -> cache slot of one rank, least recently used evicted first."""

    def __init__(self, n_slots: int):
        if n_slots < 1:
            raise ValueError("n_slots must be positive")
        self.n_slots = n_slots
        self._slot = collections.OrderedDict()   # user -> slot, oldest use first
        self._free = list(range(n_slots - 1, -1, -1))

    def __contains__(self, user: int) -> bool:
        return user in self._slot

    def lookup(self, users: Sequence[int]) -> List[int]:
        """Slots of users that hold a cached sequence (KeyError otherwise); marks them used."""
        out = []
        for u in users:
            s = self._slot[u]
            self._slot.move_to_end(u)
            out.append(s)
        return out

    def assign(self, users: Sequence[int]) -> List[int]:
        """Slots for `users` (distinct): a user already present keeps its slot,
        a new one takes a free slot or the least recently used one outside
        this batch.  Evicted users lose their cached sequence."""
        if len(set(users)) != len(users):
            raise ValueError("a user appears twice in one batch")
        if len(users) > self.n_slots:
            raise ValueError("more users in one batch than cache slots")
        batch = set(users)
        out = []
        for u in users:
            if u in self._slot:
                self._slot.move_to_end(u)
                out.append(self._slot[u])
                continue
            if self._free:
                s = self._free.pop()
            else:
                victim = next(v for v in self._slot if v not in batch)
                s = self._slot.pop(victim)
            self._slot[u] = s
            out.append(s)
        return out

    def evict(self, user: int) -> None:
        self._free.append(self._slot.pop(user))


class ReplicaShard:
    """One rank's replica: the model, a cache of `n_slots` users of up to
    `max_L_S` S tokens, and the slot table.  Every user passed in must be
    owned by this rank (`owner_rank(user, world) == rank`)."""

    def __init__(self, model: Model, n_slots: int, max_L_S: int, rank: int = 0, world: int = 1):
        self.model, self.rank, self.world = model, rank, world
        self.cache = Cache(model, n_slots, max_L_S)
        self.slots = SlotTable(n_slots)
        self._ws = torch.empty(256, dtype=torch.uint8, device="cuda")

    def _own(self, users: Sequence[int]) -> None:
        for u in users:
            if owner_rank(u, self.world) != self.rank:
                raise ValueError(f"user {u} belongs to rank {owner_rank(u, self.world)}, not {self.rank}")

    def _workspace(self, op: int, n: int, L: int) -> torch.Tensor:
        need = self.model.workspace_size(op, n, L)
        if need > self._ws.numel():
            self._ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        return self._ws

    def encode(self, users: Sequence[int], s_tokens: torch.Tensor, stream=None) -> None:
        """Stage I of the users' S tokens [U, L_S, d] into their slots."""
        self._own(users)
        slots = self.slots.assign(users)
        U, L_S, _ = s_tokens.shape
        onetrans_stage1_encode(self.model, self.cache, slots, s_tokens, self._workspace(OP_STAGE1, U, L_S), stream)

    def append(self, users: Sequence[int], events: torch.Tensor, types: torch.Tensor, stream=None) -> None:
        """Cross-request append of dL events [U, dL, e] (types [U, dL] int32) to cached users."""
        self._own(users)
        slots = self.slots.lookup(users)
        onetrans_cache_append(self.model, self.cache, slots, events, types,
                              self._workspace(OP_APPEND, len(users), events.shape[1]), stream)

    def score(self, users: Sequence[int], cand_offsets: Sequence[int], ns_tokens: torch.Tensor,
              ns_out: torch.Tensor, logits: Optional[torch.Tensor] = None, stream=None) -> None:
        """Stage II of the candidates of cached users (CSR offsets, as onetrans_stage2_score)."""
        self._own(users)
        slots = self.slots.lookup(users)
        max_len = max(self.cache.length(s) for s in slots) if slots else 0
        onetrans_stage2_score(self.model, self.cache, slots, cand_offsets, ns_tokens, ns_out,
                              self._workspace(OP_STAGE2, int(cand_offsets[-1]), max_len), stream, logits=logits)


def gather_to_rank0(user_ids: Sequence[int], values: torch.Tensor, group=None):
    """Collect every rank's (user ids, per-user values) on rank 0: a dict
    user id -> values row there, None on the other ranks.  The one exchange
    of the sharded serving path, after scoring, off the hot path."""
    import torch.distributed as dist
    payload = (list(map(int, user_ids)), values.detach().cpu())
    if not (dist.is_available() and dist.is_initialized()):
        return {u: payload[1][i] for i, u in enumerate(payload[0])}
    world = dist.get_world_size(group)
    got = [None] * world if dist.get_rank(group) == 0 else None
    dist.gather_object(payload, got, dst=0, group=group)
    if got is None:
        return None
    out = {}
    for ids, vals in got:
        for i, u in enumerate(ids):
            out[u] = vals[i]
    return out
