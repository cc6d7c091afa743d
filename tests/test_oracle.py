"""Pins of the fp64 oracle against things other than itself.

Each test ties one part of the oracle to a library routine, a closed form, a
special case, an invariant the pages state, or a worked answer the pages print.
Sources: fun-rec mdbook 7.5 "OneTrans: Unifying Sequence Modeling and Feature
Interaction" ([FR]).
"""
import copy
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from onetrans_synth import (ModelShape, WORKLOADS, bf16_round, gen_normal,
                            linear_pyramid, make_group_weights, make_weights,
                            random_types, tiny_raw_inputs)
from oracle import flops, onetrans as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
EPS = 1e-6


def small_model(n_layers=2, d=32, H=2, dff=64, L_NS=3, seed=7):
    shape = ModelShape(n_layers=n_layers, d=d, n_heads=H, d_ff=dff, L_NS=L_NS,
                       ns_feat=24, ns_hidden=L_NS * d, behavior_dims=(8, 12, 16))
    # larger weights than the workloads use, so attention is far from uniform
    return shape, make_weights(shape, seed, "fp32", std=0.2)


def t64(a):
    return torch.as_tensor(np.asarray(a, dtype=np.float64))


# ---------------------------------------------------------------- elementwise

def test_rmsnorm_matches_torch():
    x = gen_normal(1, (5, 32), "fp32", std=3.0)
    g = gen_normal(2, (32,), "fp32", mean=1.0, std=0.3)
    ref = F.rms_norm(t64(x), (32,), t64(g), eps=EPS).numpy()
    np.testing.assert_allclose(O.rmsnorm(x, g, EPS), ref, rtol=1e-13, atol=1e-13)


def test_gelu_tanh_matches_torch():
    x = np.linspace(-8, 8, 1001)
    ref = F.gelu(t64(x), approximate="tanh").numpy()
    np.testing.assert_allclose(O.gelu_tanh(x), ref, rtol=1e-13, atol=1e-15)


def test_bf16_round_matches_torch():
    x = gen_normal(3, (4096,), "fp32", std=10.0)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(bf16_round(x), ref)


# ------------------------------------------------------------------ attention

def test_attention_matches_sdpa_with_mask():
    rng = np.random.default_rng(0)
    Lq, Lk, d, H = 5, 9, 16, 2
    q, k, v = rng.standard_normal((Lq, d)), rng.standard_normal((Lk, d)), rng.standard_normal((Lk, d))
    q_pos = np.array([0, 2, 4, 7, 8])
    out = O.masked_attention(q, k, v, q_pos, H)
    mask = torch.arange(Lk)[None, :] <= torch.as_tensor(q_pos)[:, None]
    dh = d // H
    qt = t64(q).view(Lq, H, dh).transpose(0, 1)
    kt = t64(k).view(Lk, H, dh).transpose(0, 1)
    vt = t64(v).view(Lk, H, dh).transpose(0, 1)
    ref = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask).transpose(0, 1).reshape(Lq, d)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_attention_single_visible_key_returns_its_value():
    rng = np.random.default_rng(1)
    q, k, v = rng.standard_normal((1, 8)), rng.standard_normal((4, 8)), rng.standard_normal((4, 8))
    out = O.masked_attention(q, k, v, np.array([0]), 2)
    np.testing.assert_allclose(out[0], v[0], rtol=0, atol=1e-15)


def test_attention_identical_keys_average_visible_values():
    rng = np.random.default_rng(2)
    k = np.tile(rng.standard_normal((1, 8)), (6, 1))
    v = rng.standard_normal((6, 8))
    q = rng.standard_normal((3, 8))
    out = O.masked_attention(q, k, v, np.array([1, 3, 5]), 2)
    for i, p in enumerate([1, 3, 5]):
        np.testing.assert_allclose(out[i], v[: p + 1].mean(axis=0), atol=1e-14)


# --------------------------------------------------------- block and stack

def textbook_stack(X0, W, n_heads, eps):
    """A standard pre-RMSNorm causal transformer built from torch routines
    (rms_norm, linear, scaled_dot_product_attention with is_causal, gelu)."""
    x = t64(X0)
    B, L, d = x.shape
    dh = d // n_heads
    for l in range(len(W["Wo"])):
        h = F.rms_norm(x, (d,), t64(W["g_attn"][l]), eps=eps)
        Wq, Wk, Wv = (t64(W["Wqkv_S"][l][i * d:(i + 1) * d]) for i in range(3))

        def heads(t):
            return t.view(B, L, n_heads, dh).transpose(1, 2)
        a = F.scaled_dot_product_attention(heads(F.linear(h, Wq)), heads(F.linear(h, Wk)),
                                           heads(F.linear(h, Wv)), is_causal=True)
        x = x + F.linear(a.transpose(1, 2).reshape(B, L, d), t64(W["Wo"][l]))
        h2 = F.rms_norm(x, (d,), t64(W["g_ffn"][l]), eps=eps)
        f = F.linear(F.gelu(F.linear(h2, t64(W["W1_S"][l]), t64(W["b1_S"][l])), approximate="tanh"),
                     t64(W["W2_S"][l]), t64(W["b2_S"][l]))
        x = x + f
    return x.numpy()


def test_shared_ns_weights_reduce_to_textbook_transformer():
    shape, W = small_model(n_layers=2)
    W = copy.deepcopy(W)
    for l in range(shape.n_layers):
        for key, src in (("Wqkv_NS", "Wqkv_S"), ("W1_NS", "W1_S"), ("b1_NS", "b1_S"),
                         ("W2_NS", "W2_S"), ("b2_NS", "b2_S")):
            W[key][l] = np.stack([W[src][l]] * shape.L_NS)
    X0 = gen_normal(11, (2, 10 + shape.L_NS, shape.d), "fp32")
    out = O.forward(X0, W, shape.L_NS, shape.n_heads, EPS)
    ref = textbook_stack(X0, W, shape.n_heads, EPS)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-11)


def test_ns_token_weights_are_token_specific():
    """FFN weights of NS token j change only output row n_S + j; its K/V
    weights change rows n_S + j and later, never earlier rows."""
    shape, W = small_model(n_layers=1)
    n_S, j = 10, 1
    X0 = gen_normal(12, (1, n_S + shape.L_NS, shape.d), "fp32")
    base = O.forward(X0, W, shape.L_NS, shape.n_heads, EPS)[0]
    W2 = copy.deepcopy(W)
    W2["W2_NS"][0] = W2["W2_NS"][0].copy()
    W2["W2_NS"][0][j] += 0.5
    out = O.forward(X0, W2, shape.L_NS, shape.n_heads, EPS)[0]
    changed = np.abs(out - base).max(axis=1) > 1e-9
    assert changed.tolist() == [r == n_S + j for r in range(n_S + shape.L_NS)]
    W3 = copy.deepcopy(W)
    W3["Wqkv_NS"][0] = W3["Wqkv_NS"][0].copy()
    W3["Wqkv_NS"][0][j, shape.d:] += 0.5           # K and V rows of token j
    out = O.forward(X0, W3, shape.L_NS, shape.n_heads, EPS)[0]
    changed = np.abs(out - base).max(axis=1) > 1e-9
    assert changed.tolist() == [r >= n_S + j for r in range(n_S + shape.L_NS)]
    W4 = copy.deepcopy(W)
    W4["W1_S"][0] = W4["W1_S"][0] + 0.5
    out = O.forward(X0, W4, shape.L_NS, shape.n_heads, EPS)[0]
    changed = np.abs(out - base).max(axis=1) > 1e-9
    assert changed.tolist() == [r < n_S for r in range(n_S + shape.L_NS)]


def test_causality_s_rows_ignore_ns_and_later_rows():
    """[FR] 7.5.1: S rows see only earlier S rows; NS rows come after."""
    shape, W = small_model(n_layers=2)
    n_S = 9
    X0 = gen_normal(13, (1, n_S + shape.L_NS, shape.d), "fp32")
    base = O.forward(X0, W, shape.L_NS, shape.n_heads, EPS)[0]
    X1 = X0.copy()
    X1[0, n_S:] += gen_normal(14, (shape.L_NS, shape.d), "fp32")
    out = O.forward(X1, W, shape.L_NS, shape.n_heads, EPS)[0]
    np.testing.assert_array_equal(out[:n_S], base[:n_S])
    assert np.abs(out[n_S:] - base[n_S:]).max() > 1e-3
    X2 = X0.copy()
    X2[0, 5] += 1.0
    out = O.forward(X2, W, shape.L_NS, shape.n_heads, EPS)[0]
    np.testing.assert_array_equal(out[:5], base[:5])
    assert np.abs(out[5:] - base[5:]).max(axis=1).min() > 1e-9


def test_pyramid_layer_tail_equals_full_query_rows():
    """[FR] 7.5.2: queries only from the tail set; the kept rows equal the same
    rows of the full-query layer."""
    shape, W = small_model(n_layers=1)
    L = 14 + shape.L_NS
    x = gen_normal(15, (L, shape.d), "fp32")
    full = O.block(x, W, 0, shape.L_NS, L, shape.n_heads, EPS)
    for Lq in (shape.L_NS, 7, L - 1):
        tail = O.block(x, W, 0, shape.L_NS, Lq, shape.n_heads, EPS)
        np.testing.assert_allclose(tail, full[L - Lq:], rtol=1e-13, atol=1e-13)


def test_schedule_keeping_every_row_equals_no_pyramid():
    shape, W = small_model(n_layers=2)
    L0 = 8 + shape.L_NS
    X0 = gen_normal(16, (2, L0, shape.d), "fp32")
    a = O.forward(X0, W, shape.L_NS, shape.n_heads, EPS, schedule=[L0, L0])
    b = O.forward(X0, W, shape.L_NS, shape.n_heads, EPS)
    np.testing.assert_array_equal(a, b)


def test_linear_pyramid_schedule_closed_form():
    for L0, Lmin, N in ((1190, 12, 6), (2064, 16, 8), (30, 4, 3), (100, 5, 2)):
        s = linear_pyramid(L0, Lmin, N)
        assert s[0] == L0 and s[-1] == Lmin and len(s) == N
        for n in range(1, N + 1):
            drop = Fraction((L0 - Lmin) * (n - 1), N - 1)
            assert s[n - 1] == L0 - int(drop + Fraction(1, 2))   # round half up
        assert all(a > b for a, b in zip(s, s[1:]))


# ----------------------------------------------------------- two-stage path

def _check_stage_split(shape, W, L_S, schedule, seed):
    U_C = 3
    S = gen_normal(seed, (L_S, shape.d), "fp32")
    NS = gen_normal(seed + 1, (U_C, shape.L_NS, shape.d), "fp32")
    cache = O.stage1(S, W, shape.L_NS, shape.n_heads, EPS, schedule)
    for c in range(U_C):
        X0 = np.concatenate([S, NS[c]])[None]
        ref = O.forward(X0, W, shape.L_NS, shape.n_heads, EPS, schedule)[0]
        got = O.stage2(cache, NS[c], W, shape.n_heads, EPS)
        np.testing.assert_allclose(got, ref[-shape.L_NS:], rtol=1e-12, atol=1e-12)
        if schedule is None:
            np.testing.assert_allclose(got, ref[L_S:], rtol=1e-12, atol=1e-12)


def test_stage1_plus_stage2_equals_one_pass_forward():
    """[FR] 7.5.3: Stage I caches S-side K/V, Stage II scores NS rows against
    it; the result equals the unified one-pass graph."""
    shape, W = small_model(n_layers=1)
    _check_stage_split(shape, W, 11, None, 20)
    shape, W = small_model(n_layers=3, L_NS=4)
    _check_stage_split(shape, W, 16, None, 22)
    _check_stage_split(shape, W, 16, [20, 12, 4], 24)
    _check_stage_split(shape, W, 16, [17, 9, 5], 26)


def test_append_equals_full_recompute_and_zero_append_is_noop():
    """[FR] 7.5.3 cross-request caching: only the new events' K/V are computed
    and concatenated; equal to recomputing Stage I on the longer sequence."""
    shape, W = small_model(n_layers=3)
    S = gen_normal(30, (15, shape.d), "fp32")
    for dL in (1, 4):
        old = O.stage1(S[: 15 - dL], W, shape.L_NS, shape.n_heads, EPS)
        new = O.append(old, S[15 - dL:], W, shape.n_heads, EPS)
        full = O.stage1(S, W, shape.L_NS, shape.n_heads, EPS)
        for (K, V), (Kf, Vf) in zip(new, full):
            np.testing.assert_allclose(K, Kf, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(V, Vf, rtol=1e-12, atol=1e-12)
    old = O.stage1(S, W, shape.L_NS, shape.n_heads, EPS)
    same = O.append(old, S[:0], W, shape.n_heads, EPS)
    for (K, V), (Kf, Vf) in zip(same, old):
        np.testing.assert_array_equal(K, Kf)
        np.testing.assert_array_equal(V, Vf)


# -------------------------------------------------------------- tokenizers

def test_autosplit_equals_concat_mlp_reshape():
    """[FR] 7.5.0: NS-tokens = Split(MLP(Concat(NS)), L_NS)."""
    shape, W = small_model()
    groups = [gen_normal(40 + i, (5, w), "fp32") for i, w in enumerate((10, 6, 8))]
    feats = np.concatenate(groups, axis=1)
    mlp = torch.nn.Sequential(torch.nn.Linear(24, shape.ns_hidden), torch.nn.GELU("tanh"),
                              torch.nn.Linear(shape.ns_hidden, shape.L_NS * shape.d)).double()
    with torch.no_grad():
        mlp[0].weight.copy_(t64(W["Wa1"])); mlp[0].bias.copy_(t64(W["ba1"]))
        mlp[2].weight.copy_(t64(W["Wa2"])); mlp[2].bias.copy_(t64(W["ba2"]))
        ref = mlp(t64(feats)).view(5, shape.L_NS, shape.d).numpy()
    np.testing.assert_allclose(O.autosplit(feats, W, shape.L_NS), ref, rtol=1e-12, atol=1e-13)


def test_score_head_is_a_linear_unit_over_token_major_concatenation():
    """The optional head: logit = w_head . vec(h_NS) + b_head.  A one-hot
    w_head at t*d + k reads entry (t, k), which fixes the concatenation
    order (token-major); random weights match torch's linear layer over the
    row-major flattened rows."""
    shape, W = small_model()
    h = gen_normal(60, (4, shape.L_NS, shape.d), "fp32")
    W = dict(W)
    for t, k in ((0, 0), (1, 5), (shape.L_NS - 1, shape.d - 1)):
        W["w_head"] = np.zeros(shape.L_NS * shape.d)
        W["w_head"][t * shape.d + k] = 1.0
        W["b_head"] = np.array([0.25])
        np.testing.assert_array_equal(O.score_head(h, W), h[:, t, k].astype(np.float64) + 0.25)
    W["w_head"] = gen_normal(61, (shape.L_NS * shape.d,), "fp32")
    W["b_head"] = gen_normal(62, (1,), "fp32")
    ref = F.linear(t64(h).reshape(4, -1), t64(W["w_head"])[None], t64(W["b_head"]))[:, 0].numpy()
    np.testing.assert_allclose(O.score_head(h, W), ref, rtol=1e-12, atol=1e-12)


GROUP_DIMS, GROUP_HIDDEN = (10, 6, 8, 3), (12, 7, 16, 5)


def test_groupwise_tokenizer_is_one_torch_mlp_per_group():
    """[PD] 2.1, [LP] 3.1: group g through its own MLP gives NS token g."""
    d = 9
    G = make_group_weights(d, GROUP_DIMS, GROUP_HIDDEN, 60, "fp32", std=0.3)
    groups = [gen_normal(61 + g, (5, F_g), "fp32") for g, F_g in enumerate(GROUP_DIMS)]
    got = O.tokenize_groupwise(groups, G)
    assert got.shape == (5, len(GROUP_DIMS), d)
    for g, (F_g, h_g) in enumerate(zip(GROUP_DIMS, GROUP_HIDDEN)):
        mlp = torch.nn.Sequential(torch.nn.Linear(F_g, h_g), torch.nn.GELU("tanh"),
                                  torch.nn.Linear(h_g, d)).double()
        with torch.no_grad():
            mlp[0].weight.copy_(t64(G["Wg1"][g])); mlp[0].bias.copy_(t64(G["bg1"][g]))
            mlp[2].weight.copy_(t64(G["Wg2"][g])); mlp[2].bias.copy_(t64(G["bg2"][g]))
            ref = mlp(t64(groups[g])).numpy()
        np.testing.assert_allclose(got[:, g], ref, rtol=1e-12, atol=1e-13)


def test_groupwise_tokenizer_is_autosplit_with_block_diagonal_weights():
    """The two NS tokenizers of [PD] 2.1 meet: an auto-split MLP whose layers
    are block-diagonal by group (group g's inputs feed only its hidden units,
    which feed only output columns [g d, (g+1) d)) is the group-wise tokenizer,
    GELU acting elementwise.  Token order and split direction must agree."""
    from scipy.linalg import block_diag
    d = 9
    G = make_group_weights(d, GROUP_DIMS, GROUP_HIDDEN, 62, "fp32", std=0.3)
    groups = [gen_normal(63 + g, (7, F_g), "fp32") for g, F_g in enumerate(GROUP_DIMS)]
    W = {"Wa1": block_diag(*G["Wg1"]), "ba1": np.concatenate(G["bg1"]),
         "Wa2": block_diag(*G["Wg2"]), "ba2": np.concatenate(G["bg2"])}
    assert W["Wa1"].shape == (sum(GROUP_HIDDEN), sum(GROUP_DIMS))
    assert W["Wa2"].shape == (len(GROUP_DIMS) * d, sum(GROUP_HIDDEN))
    split = O.autosplit(np.concatenate(groups, axis=1), W, len(GROUP_DIMS))
    np.testing.assert_allclose(O.tokenize_groupwise(groups, G), split, rtol=1e-12, atol=1e-14)


def test_tokenize_events_per_type_mlp_plus_type_embedding():
    shape, _ = small_model()
    W = make_weights(shape, 8, "fp32", event_dim=8, std=0.2)
    ev = gen_normal(50, (2, 6, 8), "fp32")
    ty = random_types(51, (2, 6), 3)
    out = O.tokenize_events(ev, ty, W)
    for u in range(2):
        for t in range(6):
            k = int(ty[u, t])
            h = F.gelu(F.linear(t64(ev[u, t]), t64(W["Wb1"][k]), t64(W["bb1"][k])), approximate="tanh")
            ref = F.linear(h, t64(W["Wb2"][k]), t64(W["bb2"][k])) + t64(W["type_emb"][k])
            np.testing.assert_allclose(out[u, t], ref.numpy(), rtol=1e-12, atol=1e-13)


def test_intent_order_merge_length_and_sep_position():
    """[FR] 7.5.0: L_S = sum_i L_i + L_SEP, a learnable [SEP] between sequences."""
    wl = WORKLOADS["tiny"]
    W = make_weights(wl.shape, wl.seed_weights, "fp32")
    raw = tiny_raw_inputs(0)
    S = O.merge_intent_order([raw["seq0"][0], raw["seq1"][0]], W)
    assert S.shape == (wl.L_S, wl.shape.d) == (12 + 11 + 1, 32)
    np.testing.assert_array_equal(S[12], np.asarray(W["sep"], dtype=np.float64))


@pytest.mark.parametrize("lens", [(5, 0, 7), (0, 0), (9,), (3, 4, 2, 6)])
def test_intent_order_merge_rows_are_each_sequence_through_its_torch_mlp(lens):
    """Sequence i's rows are its events through behavior i's MLP (a torch
    Linear-GELU-Linear), placed after the earlier sequences and their [SEP]s;
    an empty sequence still gets its [SEP]."""
    shape, _ = small_model()
    n = len(lens)
    dims = tuple(8 + 4 * i for i in range(n))
    shape = ModelShape(n_layers=1, d=shape.d, n_heads=shape.n_heads, d_ff=shape.d_ff, L_NS=shape.L_NS,
                       ns_feat=shape.ns_feat, ns_hidden=shape.ns_hidden, behavior_dims=dims)
    W = make_weights(shape, 70, "fp32", std=0.3)
    seqs = [gen_normal(71 + i, (L, dims[i]), "fp32") for i, L in enumerate(lens)]
    S = O.merge_intent_order(seqs, W)
    assert S.shape == (sum(lens) + n - 1, shape.d)
    row = 0
    for i, x in enumerate(seqs):
        mlp = torch.nn.Sequential(torch.nn.Linear(dims[i], shape.d), torch.nn.GELU("tanh"),
                                  torch.nn.Linear(shape.d, shape.d)).double()
        with torch.no_grad():
            mlp[0].weight.copy_(t64(W["Wb1"][i])); mlp[0].bias.copy_(t64(W["bb1"][i]))
            mlp[2].weight.copy_(t64(W["Wb2"][i])); mlp[2].bias.copy_(t64(W["bb2"][i]))
            ref = mlp(t64(x)).numpy()
        np.testing.assert_allclose(S[row:row + len(x)], ref, rtol=1e-12, atol=1e-13)
        row += len(x)
        if i + 1 < n:
            np.testing.assert_array_equal(S[row], np.asarray(W["sep"], dtype=np.float64))
            row += 1
    assert row == S.shape[0]


# ------------------------------------------------------------- FLOP counter

def test_flop_counter_reproduces_worked_answers():
    g = json.load(open(os.path.join(GOLDEN, "worked_answers.json")))
    p = g["pyramid_problem_7_5_3"]
    r_fixed = flops.pyramid_attention_ratio(p["L"], p["n_layers"], shrink_keys=False)
    assert r_fixed * p["full_sum_over_L2"] == pytest.approx(p["pyramid_sum_over_L2_keys_fixed"])
    assert round(r_fixed * p["full_sum_over_L2"], 2) == p["pyramid_sum_over_L2_printed"]
    assert abs(r_fixed - p["ratio_printed"]) <= p["ratio_printed_tolerance"]
    assert flops.pyramid_attention_ratio(p["L"], p["n_layers"], shrink_keys=True) < r_fixed
    k = g["kv_cache_problem_7_5_4"]
    assert k["C"] * k["L_S"] == k["without_cache"]
    assert k["L_S"] + k["C"] * k["L_NS"] == k["with_cache"]
    assert abs(flops.kv_cache_ratio(k["C"], k["L_S"], k["L_NS"]) - k["ratio_printed"]) <= k["ratio_printed_tolerance"]


def test_flop_counter_attention_matches_brute_force_mask_count():
    """Visible (query, key) pairs counted by brute force over the mask."""
    L_S, L_NS, d, sched = 13, 3, 8, [16, 10, 3]
    f = flops.forward_flops(L_S, L_NS, d, 4 * d, 3, sched)
    L, pairs = L_S + L_NS, 0
    for Lq in sched:
        for qi in range(L - Lq, L):
            pairs += sum(1 for ki in range(L) if ki <= qi)
        L = Lq
    assert f["attn"] == 4 * d * pairs


def test_flop_counter_projections_match_torch_flop_counter():
    """Without a pyramid every row runs every projection; torch's own FLOP
    counter over the textbook stack's linear layers must give the same count."""
    from torch.utils.flop_counter import FlopCounterMode
    shape, W = small_model(n_layers=2)
    L_S = 8
    X0 = gen_normal(21, (1, L_S + shape.L_NS, shape.d), "fp32")
    with FlopCounterMode(display=False) as fc:
        textbook_stack(X0, W, shape.n_heads, EPS)
    counts = {str(k): v for k, v in fc.get_flop_counts()["Global"].items()}
    mm = counts.get("aten.mm", 0) + counts.get("aten.addmm", 0)
    f = flops.forward_flops(L_S, shape.L_NS, shape.d, shape.d_ff, shape.n_layers)
    assert f["proj"] == mm


@pytest.mark.parametrize("L_S,L_NS,N,L_min", [(13, 3, 3, 3), (40, 4, 5, 9), (7, 2, 1, 2), (30, 6, 4, None)])
def test_stage_split_flops_add_up_to_one_pass(L_S, L_NS, N, L_min):
    """[FR] 7.5.3: Stage I (S rows) plus Stage II of one candidate (NS rows)
    does exactly the one-pass work, pyramid or not (NS rows are the tail, so
    every layer keeps them).  The auto-split term is one multiply-add per
    weight entry per candidate."""
    d, d_ff, F_, H = 16, 48, 10, 24
    sched = None if L_min is None else linear_pyramid(L_S + L_NS, L_min, N)
    one = flops.forward_flops(L_S, L_NS, d, d_ff, N, sched)
    s1 = flops.stage1_flops(L_S, L_NS, d, d_ff, N, sched)
    s2 = flops.stage2_flops(L_S, L_NS, d, d_ff, N, F_, H, sched)
    assert s1["proj"] + s2["proj"] == one["proj"]
    assert s1["attn"] + s2["attn"] == one["attn"]
    assert s2["tokenize"] == 2 * (H * F_ + L_NS * d * H)   # Wa1 [H, F], Wa2 [L_NS d, H]


@pytest.mark.parametrize("L_old,dL,t", [(20, 5, 0), (1, 1, 2), (64, 17, 1)])
def test_append_flops_equal_the_grown_stage1_minus_the_old(L_old, dL, t):
    """An append of dL events costs what Stage I of the longer sequence costs
    beyond Stage I of the old one (non-pyramid); its tokenizer term is one
    multiply-add per weight entry of the event's per-behavior MLP per event."""
    shape, W = small_model(n_layers=3)
    d, N = shape.d, shape.n_layers
    e = W["Wb1"][t].shape[1]
    a = flops.append_flops(L_old, dL, d, shape.d_ff, N, e)
    grown = flops.stage1_flops(L_old + dL, shape.L_NS, d, shape.d_ff, N)
    old = flops.stage1_flops(L_old, shape.L_NS, d, shape.d_ff, N)
    assert a["proj"] == grown["proj"] - old["proj"]
    assert a["attn"] == grown["attn"] - old["attn"]
    assert a["tokenize"] == 2 * dL * (W["Wb1"][t].size + W["Wb2"][t].size)
