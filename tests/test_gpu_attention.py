"""Attention numerics at a weight scale where they decide the output.

Weights are drawn at std 1/sqrt(d): q and k entries come out ~N(0, 1) and the
scores q.k/sqrt(d_h) ~N(0, 1), so the softmax is far from uniform ([FR] 7.5.1
"Mixed Causal Attention").  At this scale the planted mistakes of
`test_oracle_sensitivity.py` (scores ignored, one future key leaked, Stage
II's own-key mask dropped) move the output by more than twice the tolerance,
so these tests fail on them; at std 0.02 the same mistakes stay inside it.

Covered, through the C ABI against the fp64 oracle (max-abs-error / RMS <=
2e-2 bf16, 1e-4 float32): forward with the pyramid, Stage I + Stage II,
append, at d = 256 (d_h 64) and d = 384 (d_h 96), on the tensor-core and
CUDA-core kernel sets; the stack's update (output minus input) at the same
tolerance; the lazy rescale of the running max (a crafted W^K = alpha W^Q
drives it, and the test checks from the oracle's own q and k that it is
driven); Stage II's mask bit for bit (no key of another candidate in the
same tile, no later NS token of the same candidate); a ragged Stage II call
with more candidate tiles than a small workspace table would hold."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from onetrans_synth import WORKLOADS, gen_normal, linear_pyramid, random_types
from oracle import onetrans as O
from helpers import (EPS, TOL, attn_std, build, rel_err, run_forward, run_stage12, shape, stored_err, tdt,
                     to_dev, to_np)

import unified_transformer_recommender_b200 as ot  # noqa: E402


@pytest.fixture(autouse=True)
def _policy_reset():
    yield
    ot.onetrans_set_kernel_policy(0)
    assert ot.onetrans_device_status() == 0


def _shape(d):
    if d == 256:
        return shape(n_layers=3)
    return shape(n_layers=2, d=384, dff=1536, L_NS=16)


MATRIX = [("bf16", 0, 256), ("bf16", 1, 256), ("fp32", 0, 256), ("bf16", 0, 384), ("bf16", 1, 384),
          ("fp32", 0, 384)]


# ------------------------------------------------------------ parity matrix

@pytest.mark.parametrize("dtype,policy,d", MATRIX)
def test_forward_pyramid_attention_scale(dtype, policy, d):
    ot.onetrans_set_kernel_policy(policy)
    sh = _shape(d)
    L_S = 290 if d == 256 else 200
    sched = linear_pyramid(L_S + sh.L_NS, sh.L_NS, sh.n_layers)
    b = build(sh, 201, dtype, pyramid=sched, std=attn_std(d))
    X0 = gen_normal(202, (3, L_S + sh.L_NS, sh.d), dtype)
    got = run_forward(b, X0)
    ref = O.forward(X0, b.W, sh.L_NS, sh.n_heads, EPS, sched)
    assert rel_err(got, ref) <= TOL[dtype]
    tail = X0[:, -sched[-1]:]
    assert rel_err(got - tail, ref - tail) <= TOL[dtype]


@pytest.mark.parametrize("dtype,policy,d", MATRIX)
def test_stage1_stage2_attention_scale(dtype, policy, d):
    """Ragged candidate counts (a user with none, one with many tiles),
    slots in a non-identity order; cached K/V page by page, then every
    candidate's final NS rows and their update."""
    ot.onetrans_set_kernel_policy(policy)
    sh = _shape(d)
    L_S = 275 if d == 256 else 200
    sched = linear_pyramid(L_S + sh.L_NS, sh.L_NS, sh.n_layers)
    b = build(sh, 203, dtype, pyramid=sched, std=attn_std(d))
    U = 3
    S = gen_normal(204, (U, L_S, sh.d), dtype)
    counts = [2, 0, 37]
    offs = np.concatenate([[0], np.cumsum(counts)]).tolist()
    NS = gen_normal(205, (offs[-1], sh.L_NS, sh.d), dtype)
    slots = [4, 0, 2]
    cache, out = run_stage12(b, S, NS, offs, slots)
    for u in range(U):
        kv = O.stage1(S[u], b.W, sh.L_NS, sh.n_heads, EPS, sched)
        for n, (K, V) in enumerate(kv):
            got = to_np(cache.gather(slots[u], n, K.shape[0]))
            assert stored_err(got[0], K, dtype) <= TOL[dtype] and stored_err(got[1], V, dtype) <= TOL[dtype], (u, n)
        for c in range(offs[u], offs[u + 1]):
            r = O.stage2(kv, NS[c], b.W, sh.n_heads, EPS)
            assert rel_err(out[c], r) <= TOL[dtype], (u, c)
            assert rel_err(out[c] - NS[c], r - NS[c]) <= TOL[dtype], (u, c)


@pytest.mark.parametrize("dtype,policy", [("bf16", 0), ("bf16", 1), ("fp32", 0)])
def test_append_attention_scale(dtype, policy):
    """Users of different cached lengths (one crossing a page boundary)
    append their events in one call; every layer's K/V and the scores after
    it against the oracle's Stage I + append of each user."""
    ot.onetrans_set_kernel_policy(policy)
    sh = shape(n_layers=2)
    b = build(sh, 206, dtype, event_dim=64, std=attn_std(sh.d))
    m = b.model
    Ls, dL, slots = [60, 45, 130], 9, [0, 2, 1]
    cache = ot.Cache(m, 3, 160)
    S = [gen_normal(207 + u, (L, sh.d), dtype) for u, L in enumerate(Ls)]
    for u, L in enumerate(Ls):
        ot.onetrans_stage1_encode(m, cache, [slots[u]], to_dev(S[u][None], tdt(dtype)),
                                  m.workspace(ot.OP_STAGE1, 1, L))
    ev = gen_normal(210, (3, dL, 64), dtype)
    ty = random_types(211, (3, dL), 3)
    ot.onetrans_cache_append(m, cache, slots, to_dev(ev, tdt(dtype)), torch.from_numpy(ty).cuda(),
                             m.workspace(ot.OP_APPEND, 3, dL))
    counts = [3, 2, 4]
    offs = np.concatenate([[0], np.cumsum(counts)]).tolist()
    NS = gen_normal(212, (offs[-1], sh.L_NS, sh.d), dtype)
    out = torch.empty(offs[-1], sh.L_NS, sh.d, dtype=torch.float32, device="cuda")
    ot.onetrans_stage2_score(m, cache, slots, offs, to_dev(NS, tdt(dtype)), out,
                             m.workspace(ot.OP_STAGE2, offs[-1], max(Ls) + dL))
    torch.cuda.synchronize()
    out = to_np(out)
    for u in range(3):
        kv = O.append(O.stage1(S[u], b.W, sh.L_NS, sh.n_heads, EPS), O.tokenize_events(ev[u], ty[u], b.W),
                      b.W, sh.n_heads, EPS)
        for n, (K, V) in enumerate(kv):
            got = to_np(cache.gather(slots[u], n, Ls[u] + dL))
            assert stored_err(got[0], K, dtype) <= TOL[dtype] and stored_err(got[1], V, dtype) <= TOL[dtype], (u, n)
        for c in range(offs[u], offs[u + 1]):
            assert rel_err(out[c], O.stage2(kv, NS[c], b.W, sh.n_heads, EPS)) <= TOL[dtype], (u, c)


@pytest.mark.parametrize("policy", [0, 1])
def test_stage2_ragged_users_many_tiles(policy):
    """Users of different cached lengths, 100 candidates each: with 12 NS
    tokens that is 30 tiles of 10 candidates, more tiles than a table sized
    for the user count alone would hold, next to the per-user key table."""
    ot.onetrans_set_kernel_policy(policy)
    sh = shape(n_layers=2)
    b = build(sh, 213, "bf16", std=attn_std(sh.d))
    m = b.model
    Ls, slots, C = [150, 97, 201], [1, 2, 0], 100
    cache = ot.Cache(m, 3, max(Ls))
    S = [gen_normal(214 + u, (L, sh.d), "bf16") for u, L in enumerate(Ls)]
    for u, L in enumerate(Ls):
        ot.onetrans_stage1_encode(m, cache, [slots[u]], to_dev(S[u][None], torch.bfloat16),
                                  m.workspace(ot.OP_STAGE1, 1, L))
    offs = [u * C for u in range(4)]
    NS = gen_normal(217, (3 * C, sh.L_NS, sh.d), "bf16")
    out = torch.empty(3 * C, sh.L_NS, sh.d, dtype=torch.float32, device="cuda")
    ot.onetrans_stage2_score(m, cache, slots, offs, to_dev(NS, torch.bfloat16), out,
                             m.workspace(ot.OP_STAGE2, 3 * C, max(Ls)))
    torch.cuda.synchronize()
    out = to_np(out)
    for u in range(3):
        kv = O.stage1(S[u], b.W, sh.L_NS, sh.n_heads, EPS)
        for c in range(offs[u], offs[u + 1]):
            assert rel_err(out[c], O.stage2(kv, NS[c], b.W, sh.n_heads, EPS)) <= TOL["bf16"], (u, c)


@pytest.mark.parametrize("dtype,policy", [("bf16", 0), ("bf16", 1), ("fp32", 0)])
def test_stage2_scoring_head(dtype, policy):
    """Stage II with the optional head (logit = w_head . vec(final NS rows) +
    b_head): against the oracle's head on its own Stage II output, and against
    the GPU's own final rows dotted on the host in fp64, which leaves only the
    kernel's fp32 summation order."""
    ot.onetrans_set_kernel_policy(policy)
    sh = shape(n_layers=2)
    b = build(sh, 236, dtype, std=attn_std(sh.d))
    m = b.model
    L_S, counts = 170, [3, 46]
    S = gen_normal(237, (2, L_S, sh.d), dtype)
    offs = np.concatenate([[0], np.cumsum(counts)]).tolist()
    C = offs[-1]
    NS = gen_normal(238, (C, sh.L_NS, sh.d), dtype)
    cache = ot.Cache(m, 2, L_S)
    ot.onetrans_stage1_encode(m, cache, [0, 1], to_dev(S, tdt(dtype)), m.workspace(ot.OP_STAGE1, 2, L_S))
    out = torch.empty(C, sh.L_NS, sh.d, dtype=torch.float32, device="cuda")
    logits = torch.full((C,), float("nan"), dtype=torch.float32, device="cuda")
    ot.onetrans_stage2_score(m, cache, [0, 1], offs, to_dev(NS, tdt(dtype)), out,
                             m.workspace(ot.OP_STAGE2, C, L_S), logits=logits)
    torch.cuda.synchronize()
    got, rows = to_np(logits), to_np(out)
    w = b.W["w_head"].astype(np.float64)
    terms = rows.reshape(C, -1).astype(np.float64) * w
    own = terms.sum(axis=1) + float(b.W["b_head"][0])
    assert np.all(np.abs(got - own) <= 1e-5 * np.abs(terms).sum(axis=1) + 1e-6)
    kvs = [O.stage1(S[u], b.W, sh.L_NS, sh.n_heads, EPS) for u in range(2)]
    ref = np.array([O.score_head(O.stage2(kvs[u], NS[c], b.W, sh.n_heads, EPS), b.W)
                    for u in range(2) for c in range(offs[u], offs[u + 1])])
    assert rel_err(got, ref) <= TOL[dtype]


# ------------------------------------------------ lazy rescale of the max

RESCALE_GAP = 8.0    # the kernels raise their running max only past this many base-2 units
KEY_TILE = 128


def _scale_keys(alpha):
    """W^K = alpha W^Q for the S set and every NS set of every layer: each
    query's score against its own key is alpha |q|^2 / sqrt(d_h), far above
    its scores against other keys."""
    def tweak(W):
        for l in range(len(W["Wqkv_S"])):
            d = W["Wqkv_S"][l].shape[1]
            W["Wqkv_S"][l][d:2 * d] = alpha * W["Wqkv_S"][l][:d]
            W["Wqkv_NS"][l][:, d:2 * d] = alpha * W["Wqkv_NS"][l][:, :d]
    return tweak


def _rescale_gaps(scores, key_tiles):
    """The amounts (base-2 units) by which a key tile's max passes the running
    max, for every raise after a row's first tile, when the max is raised only
    past RESCALE_GAP.  scores: [rows, keys] in natural-log units, -inf where
    masked; key_tiles: (lo, hi) key ranges in the order the kernel visits them."""
    s2 = scores * np.log2(np.e)
    gaps = []
    for row in s2:
        m = -np.inf
        for lo, hi in key_tiles:
            t = row[lo:hi].max() if hi > lo else -np.inf
            if t > m + RESCALE_GAP:
                if m != -np.inf:
                    gaps.append(t - m)
                m = t
    return gaps


@pytest.mark.parametrize("dtype,policy,alpha", [("bf16", 0, 1.0), ("bf16", 0, 32.0), ("bf16", 1, 32.0),
                                                ("fp32", 0, 32.0)])
def test_rescale_of_running_max_forward(dtype, policy, alpha):
    """One layer over 300 + 12 rows without a pyramid.  With alpha = 1 the own
    key's score passes the earlier tiles' maxima by just over the gap in about
    240 (row, head) pairs; with alpha = 32 nearly every row past the first key
    tile is raised, most of them by more than 128 base-2 units, where 2^gap
    overflows float32 if the rescale is skipped.  The input's rescale counts
    are computed here from the oracle's own q and k."""
    ot.onetrans_set_kernel_policy(policy)
    sh = shape(n_layers=1)
    L_S = 300
    b = build(sh, 218, dtype, std=attn_std(sh.d), tweak=_scale_keys(alpha))
    X0 = gen_normal(219, (2, L_S + sh.L_NS, sh.d), dtype)
    # the inputs drive the rescale: computed from the oracle's own q and k
    L = L_S + sh.L_NS
    h = O.rmsnorm(X0[0], b.W["g_attn"][0], EPS)
    q, k, _ = O.qkv_rows(h, b.W, 0, L_S, range(L))
    dh = sh.d_h
    tiles = [(t, min(t + KEY_TILE, L)) for t in range(0, L, KEY_TILE)]
    vis = np.arange(L)[None, :] <= np.arange(L)[:, None]
    gaps = np.array(sum((_rescale_gaps(np.where(vis, q[:, hh * dh:(hh + 1) * dh] @ k[:, hh * dh:(hh + 1) * dh].T
                                                / np.sqrt(dh), -np.inf), tiles) for hh in range(sh.n_heads)), []))
    if alpha < 2:
        assert len(gaps) >= 100, len(gaps)
    else:
        assert (gaps > 128).sum() >= 500, gaps
    got = run_forward(b, X0)
    assert np.isfinite(got).all()
    ref = O.forward(X0, b.W, sh.L_NS, sh.n_heads, EPS)
    assert rel_err(got, ref) <= TOL[dtype]
    assert rel_err(got - X0, ref - X0) <= TOL[dtype]


@pytest.mark.parametrize("dtype,policy,alpha", [("bf16", 0, 1.0), ("bf16", 0, 32.0), ("bf16", 1, 32.0)])
def test_rescale_of_running_max_stage2(dtype, policy, alpha):
    """Stage II with W^K = alpha W^Q in every NS set: the own NS key, in the
    tile after the cached S keys, passes their maximum by more than the gap."""
    ot.onetrans_set_kernel_policy(policy)
    sh = shape(n_layers=1)
    L_S = 200
    b = build(sh, 220, dtype, std=attn_std(sh.d), tweak=_scale_keys(alpha))
    S = gen_normal(221, (1, L_S, sh.d), dtype)
    NS = gen_normal(222, (23, sh.L_NS, sh.d), dtype)
    kv = O.stage1(S[0], b.W, sh.L_NS, sh.n_heads, EPS)
    K_s = kv[0][0]
    h = O.rmsnorm(NS[0], b.W["g_attn"][0], EPS)
    y = np.stack([b.W["Wqkv_NS"][0][j].astype(np.float64) @ h[j] for j in range(sh.L_NS)])
    d, dh = sh.d, sh.d_h
    q, k = y[:, :d], y[:, d:2 * d]
    keys = np.concatenate([K_s, k])
    tiles = [(t, min(t + KEY_TILE, L_S)) for t in range(0, L_S, KEY_TILE)] + [(L_S, L_S + sh.L_NS)]
    vis = np.arange(L_S + sh.L_NS)[None, :] <= (L_S + np.arange(sh.L_NS))[:, None]
    gaps = np.array(sum((_rescale_gaps(np.where(vis, q[:, hh * dh:(hh + 1) * dh] @ keys[:, hh * dh:(hh + 1) * dh].T
                                                / np.sqrt(dh), -np.inf), tiles) for hh in range(sh.n_heads)), []))
    if alpha < 2:
        assert len(gaps) >= 10, len(gaps)
    else:
        assert (gaps > 128).sum() >= 30, gaps
    _, out = run_stage12(b, S, NS, [0, 23])
    assert np.isfinite(out).all()
    for c in range(23):
        r = O.stage2(kv, NS[c], b.W, sh.n_heads, EPS)
        assert rel_err(out[c], r) <= TOL[dtype], c
        assert rel_err(out[c] - NS[c], r - NS[c]) <= TOL[dtype], c


# ------------------------------------------------------ masks, bit for bit

@pytest.mark.parametrize("policy,d", [(0, 256), (1, 256), (0, 384)])
def test_stage2_mask_exact(policy, d):
    """Candidates of one user share Stage II's query tiles (10 per tile at 12
    NS tokens, 8 at 16).  Replacing candidate c's NS inputs leaves every other
    candidate bit-identical, its own neighbours in the tile included; replacing
    its tokens j+1.. leaves its tokens 0..j bit-identical."""
    ot.onetrans_set_kernel_policy(policy)
    sh = _shape(d)
    sh = shape(n_layers=2, d=sh.d, dff=sh.d_ff, L_NS=sh.L_NS)
    L_S = 150
    b = build(sh, 223, "bf16", std=attn_std(d))
    S = gen_normal(224, (1, L_S, sh.d), "bf16")
    C, c, j = 25, 14, 5
    NS0 = gen_normal(225, (C, sh.L_NS, sh.d), "bf16")
    cache, base = run_stage12(b, S, NS0, [0, C])

    def score(NS):
        out = torch.empty(C, sh.L_NS, sh.d, dtype=torch.float32, device="cuda")
        ot.onetrans_stage2_score(b.model, cache, [0], [0, C], to_dev(NS, torch.bfloat16), out,
                                 b.model.workspace(ot.OP_STAGE2, C, L_S))
        torch.cuda.synchronize()
        return to_np(out)

    np.testing.assert_array_equal(score(NS0), base)            # deterministic
    NS1 = NS0.copy()
    NS1[c] = gen_normal(226, (sh.L_NS, sh.d), "bf16")
    out1 = score(NS1)
    others = [i for i in range(C) if i != c]
    np.testing.assert_array_equal(out1[others], base[others])
    assert (out1[c] != base[c]).any(axis=-1).all()
    NS2 = NS0.copy()
    NS2[c, j + 1:] = gen_normal(227, (sh.L_NS - j - 1, sh.d), "bf16")
    out2 = score(NS2)
    np.testing.assert_array_equal(out2[others], base[others])
    np.testing.assert_array_equal(out2[c, :j + 1], base[c, :j + 1])
    assert (out2[c, j + 1:] != base[c, j + 1:]).any(axis=-1).all()


@pytest.mark.parametrize("policy,d", [(0, 256), (1, 256), (0, 384)])
def test_causal_mask_exact_attention_scale(policy, d):
    """Perturbing the NS inputs leaves every S output row bit-identical, and
    perturbing S row t leaves rows < t bit-identical, on both kernel sets and
    both head widths."""
    ot.onetrans_set_kernel_policy(policy)
    sh = _shape(d)
    sh = shape(n_layers=2, d=sh.d, dff=sh.d_ff, L_NS=sh.L_NS)
    b = build(sh, 228, "bf16", std=attn_std(d))
    L_S = 150
    X0 = gen_normal(229, (2, L_S + sh.L_NS, sh.d), "bf16")
    base = run_forward(b, X0)
    X1 = X0.copy()
    X1[:, L_S:] = gen_normal(230, (2, sh.L_NS, sh.d), "bf16")
    out1 = run_forward(b, X1)
    np.testing.assert_array_equal(out1[:, :L_S], base[:, :L_S])
    assert np.abs(out1[:, L_S:] - base[:, L_S:]).max() > 0
    for t in (97, 128, 129):
        X2 = X0.copy()
        X2[:, t] += 1.0
        out2 = run_forward(b, X2)
        np.testing.assert_array_equal(out2[:, :t], base[:, :t])
        assert (out2[:, t] != base[:, t]).any()


# ----------------------------------------- full-size workloads, sampled

def test_kv_serving_full_size_attention_scale():
    """The serving workload's shapes (16 users x 1178 S rows, 512 candidates
    each, 6 layers, pyramid 1190 -> 12) with weights at std 1/16; sampled
    users and candidates against the oracle."""
    wl = WORKLOADS["kv_serving"]
    sh, U, C = wl.shape, wl.users, wl.cands
    b = build(sh, 231, "bf16", pyramid=list(wl.pyramid), std=attn_std(sh.d))
    S = gen_normal(232, (U, wl.L_S, sh.d), "bf16")
    NS = gen_normal(233, (U * C, sh.L_NS, sh.d), "bf16")
    _, out = run_stage12(b, S, NS, [u * C for u in range(U + 1)])
    for u in (0, U - 1):
        kv = O.stage1(S[u], b.W, sh.L_NS, sh.n_heads, EPS, wl.pyramid)
        for c in (u * C, u * C + 317, u * C + C - 1):
            r = O.stage2(kv, NS[c], b.W, sh.n_heads, EPS)
            assert rel_err(out[c], r) <= TOL["bf16"], (u, c)
            assert rel_err(out[c] - NS[c], r - NS[c]) <= TOL["bf16"], (u, c)


@pytest.mark.parametrize("name", ["s_forward", "l_forward"])
def test_forward_full_size_attention_scale(name):
    wl = WORKLOADS[name]
    sh = wl.shape
    b = build(sh, 234, "bf16", pyramid=list(wl.pyramid), std=attn_std(sh.d))
    X0 = gen_normal(235, (wl.users, wl.L0, sh.d), "bf16")
    got = run_forward(b, X0)
    u = wl.users - 1
    ref = O.forward(X0[u:u + 1], b.W, sh.L_NS, sh.n_heads, EPS, wl.pyramid)[0]
    assert rel_err(got[u], ref) <= TOL["bf16"]
    tail = X0[u, -sh.L_NS:]
    assert rel_err(got[u] - tail, ref - tail) <= TOL["bf16"]
