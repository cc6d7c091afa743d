"""One rank's replica (the whole path on one GPU): Stage I, append and Stage
II through the slot table give, bit for bit, what the direct C ABI calls on
the same slots give; a user evicted for a new one must be encoded again."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from onetrans_synth import gen_normal, random_types
from helpers import attn_std, build, shape, to_dev

import unified_transformer_recommender_b200 as ot  # noqa: E402
from unified_transformer_recommender_b200 import serving  # noqa: E402


def test_replica_shard_matches_direct_calls_and_evicts_lru():
    sh = shape(n_layers=2)
    b = build(sh, 260, "bf16", event_dim=64, std=attn_std(sh.d))
    m = b.model
    users, L_S, C = [101, 7, 55], 90, 4
    S = to_dev(gen_normal(261, (3, L_S, sh.d), "bf16"), torch.bfloat16)
    ev = to_dev(gen_normal(262, (3, 5, 64), "bf16"), torch.bfloat16)
    ty = torch.from_numpy(random_types(263, (3, 5), 3)).cuda()
    NS = to_dev(gen_normal(264, (3 * C, sh.L_NS, sh.d), "bf16"), torch.bfloat16)
    offs = [0, C, 2 * C, 3 * C]
    shard = serving.ReplicaShard(m, n_slots=3, max_L_S=128)
    shard.encode(users, S)
    shard.append(users, ev, ty)
    out = torch.empty(3 * C, sh.L_NS, sh.d, dtype=torch.float32, device="cuda")
    logits = torch.empty(3 * C, dtype=torch.float32, device="cuda")
    shard.score(users, offs, NS, out, logits)
    # the same calls made directly on the slots the table chose
    slots = shard.slots.lookup(users)
    cache = ot.Cache(m, 3, 128)
    ot.onetrans_stage1_encode(m, cache, slots, S, m.workspace(ot.OP_STAGE1, 3, L_S))
    ot.onetrans_cache_append(m, cache, slots, ev, ty, m.workspace(ot.OP_APPEND, 3, 5))
    ref = torch.empty_like(out)
    ref_logits = torch.empty_like(logits)
    ot.onetrans_stage2_score(m, cache, slots, offs, NS, ref, m.workspace(ot.OP_STAGE2, 3 * C, L_S + 5),
                             logits=ref_logits)
    torch.cuda.synchronize()
    assert torch.equal(out, ref) and torch.equal(logits, ref_logits)
    # a fourth user takes the least recently used slot
    shard.score([7, 55], [0, C, 2 * C], NS[C:], out[C:])
    shard.encode([999], S[:1])
    assert 101 not in shard.slots and 999 in shard.slots
    with pytest.raises(KeyError):
        shard.score([101], [0, C], NS[:C], out[:C])
    with pytest.raises(ValueError):
        serving.ReplicaShard(m, 2, 64, rank=0, world=2).encode(
            [u for u in range(50) if serving.owner_rank(u, 2) == 1][:1], S[:1])
    assert ot.onetrans_device_status() == 0
