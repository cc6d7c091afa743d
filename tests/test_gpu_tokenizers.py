"""S-side tokenizer, timestamp-agnostic merge (OneTrans, [FR] 7.5.0: sequences
in intent order, each through its behavior's MLP, one learnable [SEP]
between consecutive ones), through the C ABI against the fp64 oracle on the
same seeded inputs.  Token rows: max-abs-error / RMS(oracle) <= 2e-2 for bf16
storage, <= 1e-4 in float32; [SEP] rows are copies and must match bit for
bit; the layout (row of every sequence and separator) is checked exactly."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from onetrans_synth import gen_normal
from oracle import onetrans as O
from helpers import TOL, build, rel_err, shape, stored_err, to_dev, to_np

import unified_transformer_recommender_b200 as ot  # noqa: E402


def tdt(dtype):
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def by_sequence(W, seq_type):
    """The oracle applies MLP i to sequence i: give it the behavior MLPs in the
    sequences' order."""
    V = dict(W)
    for f in ("Wb1", "bb1", "Wb2", "bb2"):
        V[f] = [W[f][t] for t in seq_type]
    return V


@pytest.mark.parametrize("dtype,d,lens,types", [
    ("bf16", 256, [40, 0, 23], [0, 1, 2]),      # tiled kernel, an empty sequence in the middle
    ("fp32", 256, [70, 33, 5], [2, 0, 1]),      # intent order differs from the behavior ids
    ("bf16", 128, [10, 20], [1, 1]),            # per-event kernel, two sequences of one behavior
    ("bf16", 256, [37], [2]),                   # one sequence: no [SEP]
    ("fp32", 256, [0, 0, 0], [0, 1, 2]),        # empty sequences: only the two [SEP] rows
])
def test_merge_intent_order_matches_oracle(dtype, d, lens, types):
    sh = shape(n_layers=1, d=d, H=d // 64)
    b = build(sh, 131, dtype, event_dim=64)
    R, n = sum(lens), len(lens)
    ev = gen_normal(132, (max(R, 1), 64), dtype)[:R]
    L_S = R + n - 1
    tok = torch.full((L_S, d), float("nan"), dtype=tdt(dtype), device="cuda")
    sep = to_dev(b.W["sep"], tdt(dtype))
    ot.onetrans_merge_intent_order(b.model, to_dev(ev, tdt(dtype)) if R else None, lens, types,
                                   sep if n > 1 else None, tok)
    torch.cuda.synchronize()
    assert ot.onetrans_device_status() == 0
    seqs, r = [], 0
    for L in lens:
        seqs.append(ev[r:r + L])
        r += L
    ref = O.merge_intent_order(seqs, by_sequence(b.W, types))
    assert ref.shape == (L_S, d)
    got = to_np(tok)
    assert not np.isnan(got).any()                 # every row written
    row, sep_rows, tok_rows = 0, [], []
    for i, L in enumerate(lens):
        tok_rows += list(range(row, row + L))
        row += L
        if i + 1 < n:
            sep_rows.append(row)
            row += 1
    assert row == L_S
    for s in sep_rows:
        assert torch.equal(tok[s], sep), s
    if tok_rows:
        assert stored_err(got[tok_rows], ref[tok_rows], dtype) <= TOL[dtype]


def test_merge_of_one_sequence_is_the_event_tokenizer_without_identifier():
    """One sequence of behavior t through the merge equals the per-event
    tokenizer's output for type t minus that type's identifier row."""
    sh = shape(n_layers=1)
    b = build(sh, 133, "fp32", event_dim=64)
    L, t = 45, 1
    ev = to_dev(gen_normal(134, (L, 64), "fp32"), torch.float32)
    merged = torch.empty(L, sh.d, dtype=torch.float32, device="cuda")
    ot.onetrans_merge_intent_order(b.model, ev, [L], [t], None, merged)
    plain = torch.empty_like(merged)
    ot.onetrans_tokenize_events(b.model, ev, torch.full((L,), t, dtype=torch.int32, device="cuda"), plain)
    torch.cuda.synchronize()
    assert ot.onetrans_device_status() == 0
    emb = to_dev(b.W["type_emb"][t], torch.float32)
    torch.testing.assert_close(merged + emb, plain, rtol=0, atol=1e-5)


def pad_groups(groups, G, N, F_max, dtype):
    """[N, G, F_max] with group g's features in its first F_g columns, zeros after."""
    out = np.zeros((N, G, F_max), dtype=np.float32)
    for g, x in enumerate(groups):
        out[:, g, :x.shape[1]] = x
    return to_dev(out, tdt(dtype))


def pad_weights(Gw, d, F_max, h_max, dtype):
    G = len(Gw["Wg1"])
    W1 = np.zeros((G, h_max, F_max), np.float32); b1 = np.zeros((G, h_max), np.float32)
    W2 = np.zeros((G, d, h_max), np.float32); b2 = np.zeros((G, d), np.float32)
    for g in range(G):
        h_g, F_g = Gw["Wg1"][g].shape
        W1[g, :h_g, :F_g] = Gw["Wg1"][g]; b1[g, :h_g] = Gw["bg1"][g]
        W2[g, :, :h_g] = Gw["Wg2"][g]; b2[g] = Gw["bg2"][g]
    return [to_dev(a, tdt(dtype)) for a in (W1, b1, W2, b2)]


@pytest.mark.parametrize("dtype,dims,hidden", [
    ("bf16", (24, 40, 16, 8), (32, 64, 48, 16)),     # F_max = 40: CUDA-core up-projection, tensor-core down
    ("bf16", (64, 64, 32, 64), (128, 96, 128, 64)),  # F_max = 64, h_max = 128: tensor cores both
    ("fp32", (24, 40, 16, 8), (32, 64, 48, 16)),
])
def test_tokenize_groupwise_matches_oracle(dtype, dims, hidden):
    from onetrans_synth import make_group_weights
    G = len(dims)
    sh = shape(n_layers=1, L_NS=G)
    b = build(sh, 141, dtype)
    N, F_max, h_max = 300, max(dims), max(hidden)
    Gw = make_group_weights(sh.d, dims, hidden, 142, dtype, std=0.1)
    groups = [gen_normal(143 + g, (N, F_g), dtype) for g, F_g in enumerate(dims)]
    feats = pad_groups(groups, G, N, F_max, dtype)
    W1, b1, W2, b2 = pad_weights(Gw, sh.d, F_max, h_max, dtype)
    tok = torch.full((N, G, sh.d), float("nan"), dtype=tdt(dtype), device="cuda")
    ws = b.model.workspace(ot.OP_GROUPWISE, N, h_max)
    ot.onetrans_tokenize_groupwise(b.model, feats, W1, b1, W2, b2, tok, ws)
    torch.cuda.synchronize()
    assert ot.onetrans_device_status() == 0
    ref = O.tokenize_groupwise(groups, Gw)
    got = to_np(tok)
    assert not np.isnan(got).any()
    assert stored_err(got, ref, dtype) <= TOL[dtype]
