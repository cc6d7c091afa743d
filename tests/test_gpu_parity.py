"""CUDA path (through the C ABI) against the fp64 oracle on the same seeded
inputs.  Tolerance: max-abs-error / RMS(oracle output) <= 2e-2 for bf16
storage, <= 1e-4 in the float32 mode.  Integer parts (schedule, cache
indexing, the causal predicate) are checked exactly."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from onetrans_synth import (WORKLOADS, gen_normal, linear_pyramid, random_types,
                            tiny_raw_inputs)
from oracle import onetrans as O
from helpers import EPS, TOL, build, rel_err, run_forward, run_stage12, shape, stored_err, tdt, to_dev, to_np

import unified_transformer_recommender_b200 as ot  # noqa: E402


@pytest.fixture(autouse=True)
def _policy_reset():
    yield
    ot.onetrans_set_kernel_policy(0)
    assert ot.onetrans_device_status() == 0


# ------------------------------------------------------------------ tiny --

def test_tiny_fp32_end_to_end():
    """Tiny workload: intent-order merged S (2 sequences + [SEP]), auto-split
    NS tokens, one layer, 2 users x 3 candidates, float32 mode."""
    wl = WORKLOADS["tiny"]
    sh = wl.shape
    b = build(sh, wl.seed_weights, "fp32")
    raw = tiny_raw_inputs(wl.seed_inputs)
    U, C = wl.users, wl.cands
    S = np.stack([O.merge_intent_order([raw["seq0"][u], raw["seq1"][u]], b.W) for u in range(U)]).astype(np.float32)
    feats = raw["feats"]
    ns = torch.empty(U * C, sh.L_NS, sh.d, dtype=torch.float32, device="cuda")
    ot.onetrans_tokenize_autosplit(b.model, to_dev(feats, torch.float32), ns,
                                   b.model.workspace(ot.OP_AUTOSPLIT, U * C))
    torch.cuda.synchronize()
    ns_ref = O.autosplit(feats, b.W, sh.L_NS)                    # [N, L_NS, d], oracle's own
    assert rel_err(to_np(ns), ns_ref) <= TOL["fp32"]
    # each side runs the stack on its own tokens: GPU tokens -> GPU, oracle tokens -> oracle
    X0_gpu = torch.cat([torch.from_numpy(S).cuda()[torch.arange(U * C) // C], ns], dim=1).contiguous()
    X0_ref = np.stack([np.concatenate([S[c // C], ns_ref[c]]) for c in range(U * C)])
    out_f = torch.empty(U * C, S.shape[1] + sh.L_NS, sh.d, dtype=torch.float32, device="cuda")
    ot.onetrans_forward(b.model, X0_gpu, out_f, b.model.workspace(ot.OP_FORWARD, U * C, S.shape[1]))
    torch.cuda.synchronize()
    ref = O.forward(X0_ref, b.W, sh.L_NS, sh.n_heads, EPS)
    assert rel_err(to_np(out_f), ref) <= TOL["fp32"]
    m = b.model
    cache = ot.Cache(m, U, S.shape[1])
    ot.onetrans_stage1_encode(m, cache, [0, 1], torch.from_numpy(S).cuda(), m.workspace(ot.OP_STAGE1, U, S.shape[1]))
    out = torch.empty(U * C, sh.L_NS, sh.d, dtype=torch.float32, device="cuda")
    ot.onetrans_stage2_score(m, cache, [0, 1], [0, C, 2 * C], ns, out, m.workspace(ot.OP_STAGE2, U * C, S.shape[1]))
    torch.cuda.synchronize()
    out = to_np(out)
    for c in range(U * C):
        kv = O.stage1(S[c // C], b.W, sh.L_NS, sh.n_heads, EPS)
        r = O.stage2(kv, ns_ref[c], b.W, sh.n_heads, EPS)
        assert rel_err(out[c], r) <= TOL["fp32"]
        assert rel_err(out[c], ref[c, -sh.L_NS:]) <= TOL["fp32"]


# ------------------------------------------------------- small, bf16/fp32 --

@pytest.mark.parametrize("dtype,policy", [("bf16", 0), ("bf16", 1), ("fp32", 0)])
def test_forward_pyramid_small(dtype, policy):
    ot.onetrans_set_kernel_policy(policy)
    sh = shape(n_layers=3)
    L_S = 290
    sched = [302, 170, 12]
    b = build(sh, 101, dtype, pyramid=sched)
    X0 = gen_normal(5, (3, L_S + sh.L_NS, sh.d), dtype)
    got = run_forward(b, X0)
    ref = O.forward(X0, b.W, sh.L_NS, sh.n_heads, EPS, sched)
    assert got.shape == ref.shape == (3, 12, sh.d)
    assert rel_err(got, ref) <= TOL[dtype]
    # the layer updates themselves (output minus the rows it started from)
    assert rel_err(got - X0[:, -12:], ref - X0[:, -12:]) <= 10 * TOL[dtype]


@pytest.mark.parametrize("dtype,policy", [("bf16", 0), ("bf16", 1), ("fp32", 0)])
def test_forward_no_pyramid_keeps_all_rows(dtype, policy):
    ot.onetrans_set_kernel_policy(policy)
    sh = shape(n_layers=2)
    b = build(sh, 102, dtype)
    X0 = gen_normal(6, (2, 140 + sh.L_NS, sh.d), dtype)
    got = run_forward(b, X0)
    ref = O.forward(X0, b.W, sh.L_NS, sh.n_heads, EPS)
    assert rel_err(got, ref) <= TOL[dtype]


@pytest.mark.parametrize("dtype,policy", [("bf16", 0), ("bf16", 1), ("fp32", 0)])
def test_stage1_stage2_small_ragged(dtype, policy):
    """Ragged candidate counts (including a user with none) and slots in a
    non-identity order; cache rows read back page by page."""
    ot.onetrans_set_kernel_policy(policy)
    sh = shape(n_layers=3)
    L_S = 275
    sched = [287, 150, 12]
    b = build(sh, 103, dtype, pyramid=sched)
    U = 3
    S = gen_normal(7, (U, L_S, sh.d), dtype)
    counts = [2, 0, 131]
    offs = np.concatenate([[0], np.cumsum(counts)]).tolist()
    NS = gen_normal(8, (offs[-1], sh.L_NS, sh.d), dtype)
    slots = [4, 0, 2]
    cache, out = run_stage12(b, S, NS, offs, slots)
    for u in range(U):
        kv = O.stage1(S[u], b.W, sh.L_NS, sh.n_heads, EPS, sched)
        assert cache.length(slots[u]) == L_S
        for n, (K, V) in enumerate(kv):
            got = to_np(cache.gather(slots[u], n, K.shape[0]))
            assert stored_err(got[0], K, dtype) <= TOL[dtype]
            assert stored_err(got[1], V, dtype) <= TOL[dtype]
        for c in range(offs[u], offs[u + 1]):
            r = O.stage2(kv, NS[c], b.W, sh.n_heads, EPS)
            assert rel_err(out[c], r) <= TOL[dtype], (u, c)


@pytest.mark.parametrize("dtype,policy,pyr", [("bf16", 0, None), ("bf16", 0, [150, 80, 12]),
                                              ("bf16", 1, None), ("fp32", 0, None)])
def test_stage2_users_of_different_lengths(dtype, policy, pyr):
    """Users encoded by separate Stage I calls with different S lengths are
    scored in one Stage II call; each user's layers see its own cached keys
    (all layers without a pyramid, layer 0 with a fixed-count pyramid)."""
    ot.onetrans_set_kernel_policy(policy)
    sh = shape(n_layers=3)
    b = build(sh, 109, dtype, pyramid=pyr)
    m = b.model
    Ls = [200, 139, 257]
    slots = [2, 0, 1]
    cache = ot.Cache(m, 3, max(Ls) + 64)
    S = [gen_normal(20 + u, (L, sh.d), dtype) for u, L in enumerate(Ls)]
    for u, L in enumerate(Ls):
        ot.onetrans_stage1_encode(m, cache, [slots[u]], to_dev(S[u][None], tdt(dtype)),
                                  m.workspace(ot.OP_STAGE1, 1, L))
    counts = [5, 3, 7]
    offs = np.concatenate([[0], np.cumsum(counts)]).tolist()
    NS = gen_normal(30, (offs[-1], sh.L_NS, sh.d), dtype)
    out = torch.empty(offs[-1], sh.L_NS, sh.d, dtype=torch.float32, device="cuda")
    ot.onetrans_stage2_score(m, cache, slots, offs, to_dev(NS, tdt(dtype)), out,
                             m.workspace(ot.OP_STAGE2, offs[-1], max(Ls)))
    torch.cuda.synchronize()
    out = to_np(out)
    for u in range(3):
        assert cache.length(slots[u]) == Ls[u]
        kv = O.stage1(S[u], b.W, sh.L_NS, sh.n_heads, EPS, pyr)
        for c in range(offs[u], offs[u + 1]):
            assert rel_err(out[c], O.stage2(kv, NS[c], b.W, sh.n_heads, EPS)) <= TOL[dtype], (u, c)


@pytest.mark.parametrize("dtype,policy,pyr", [("bf16", 0, None), ("bf16", 0, [150, 80, 12]),
                                              ("bf16", 1, None), ("fp32", 0, None)])
def test_stage1_ragged_one_call(dtype, policy, pyr):
    """One Stage I call for users of different lengths (runs of equal lengths
    among them): every layer's cached K/V of every user against the oracle's
    Stage I of that user alone, then one Stage II call over all of them."""
    ot.onetrans_set_kernel_policy(policy)
    sh = shape(n_layers=3)
    b = build(sh, 151, dtype, pyramid=pyr)
    m = b.model
    Ls = [200, 200, 139, 257, 257, 140]
    slots = [4, 0, 2, 1, 5, 3]
    cache = ot.Cache(m, len(Ls), max(Ls))
    S = [gen_normal(160 + u, (L, sh.d), dtype) for u, L in enumerate(Ls)]
    packed = to_dev(np.concatenate(S, axis=0), tdt(dtype))
    ot.onetrans_stage1_encode_ragged(m, cache, slots, Ls, packed, m.workspace(ot.OP_STAGE1, len(Ls), max(Ls)))
    torch.cuda.synchronize()
    assert ot.onetrans_device_status() == 0
    kvs = []
    for u, L in enumerate(Ls):
        assert cache.length(slots[u]) == L
        kv = O.stage1(S[u], b.W, sh.L_NS, sh.n_heads, EPS, pyr)
        kvs.append(kv)
        for n, (K, V) in enumerate(kv):
            got = to_np(cache.gather(slots[u], n, K.shape[0]))
            assert stored_err(got[0], K, dtype) <= TOL[dtype] and stored_err(got[1], V, dtype) <= TOL[dtype], (u, n)
    counts = [2, 3, 1, 2, 2, 3]
    offs = np.concatenate([[0], np.cumsum(counts)]).tolist()
    NS = gen_normal(170, (offs[-1], sh.L_NS, sh.d), dtype)
    out = torch.empty(offs[-1], sh.L_NS, sh.d, dtype=torch.float32, device="cuda")
    ot.onetrans_stage2_score(m, cache, slots, offs, to_dev(NS, tdt(dtype)), out,
                             m.workspace(ot.OP_STAGE2, offs[-1], max(Ls)))
    torch.cuda.synchronize()
    out = to_np(out)
    for u in range(len(Ls)):
        for c in range(offs[u], offs[u + 1]):
            assert rel_err(out[c], O.stage2(kvs[u], NS[c], b.W, sh.n_heads, EPS)) <= TOL[dtype], (u, c)


@pytest.mark.parametrize("dtype,policy", [("bf16", 0), ("bf16", 1), ("fp32", 0)])
def test_append_users_of_different_lengths(dtype, policy):
    """One append call for users whose slots hold different lengths: each
    user's events take the positions after its own cached rows (crossing a
    page boundary for two of them); cache rows and Stage II scores against
    the oracle."""
    ot.onetrans_set_kernel_policy(policy)
    sh = shape(n_layers=2)
    b = build(sh, 111, dtype, event_dim=64)
    m = b.model
    Ls, dL, slots = [60, 45, 62], 7, [0, 2, 1]
    cache = ot.Cache(m, 3, 128)
    S = [gen_normal(40 + u, (L, sh.d), dtype) for u, L in enumerate(Ls)]
    for u, L in enumerate(Ls):
        ot.onetrans_stage1_encode(m, cache, [slots[u]], to_dev(S[u][None], tdt(dtype)),
                                  m.workspace(ot.OP_STAGE1, 1, L))
    ev = gen_normal(50, (3, dL, 64), dtype)
    ty = random_types(51, (3, dL), 3)
    ot.onetrans_cache_append(m, cache, slots, to_dev(ev, tdt(dtype)), torch.from_numpy(ty).cuda(),
                             m.workspace(ot.OP_APPEND, 3, dL))
    counts = [2, 3, 1]
    offs = np.concatenate([[0], np.cumsum(counts)]).tolist()
    NS = gen_normal(52, (offs[-1], sh.L_NS, sh.d), dtype)
    out = torch.empty(offs[-1], sh.L_NS, sh.d, dtype=torch.float32, device="cuda")
    ot.onetrans_stage2_score(m, cache, slots, offs, to_dev(NS, tdt(dtype)), out,
                             m.workspace(ot.OP_STAGE2, offs[-1], max(Ls) + dL))
    torch.cuda.synchronize()
    out = to_np(out)
    for u in range(3):
        assert cache.length(slots[u]) == Ls[u] + dL
        new = O.tokenize_events(ev[u], ty[u], b.W)
        kv = O.append(O.stage1(S[u], b.W, sh.L_NS, sh.n_heads, EPS), new, b.W, sh.n_heads, EPS)
        for n, (K, V) in enumerate(kv):
            got = to_np(cache.gather(slots[u], n, Ls[u] + dL))
            assert stored_err(got[0], K, dtype) <= TOL[dtype], (u, n)
            assert stored_err(got[1], V, dtype) <= TOL[dtype], (u, n)
        for c in range(offs[u], offs[u + 1]):
            assert rel_err(out[c], O.stage2(kv, NS[c], b.W, sh.n_heads, EPS)) <= TOL[dtype], (u, c)


@pytest.mark.parametrize("dtype,d", [("bf16", 256), ("fp32", 256), ("bf16", 128)])
def test_tokenize_events_then_stage1(dtype, d):
    """S-side tokenizer: time-ordered events of several behavior types, each
    through its type's MLP plus the type identifier, then Stage I on the
    tokens; tokens and cached K/V against the oracle.  d = 256 takes the
    tiled kernel, d = 128 the per-event one."""
    sh = shape(n_layers=2, d=d, H=d // 64)
    b = build(sh, 113, dtype, event_dim=64)
    m = b.model
    U, L = 3, 70
    ev = gen_normal(60, (U, L, 64), dtype)
    ty = random_types(61, (U, L), 3)
    tok = torch.empty(U * L, d, dtype=tdt(dtype), device="cuda")
    ot.onetrans_tokenize_events(m, to_dev(ev.reshape(U * L, 64), tdt(dtype)),
                                torch.from_numpy(ty.reshape(-1)).cuda(), tok)
    torch.cuda.synchronize()
    assert ot.onetrans_device_status() == 0
    ref = O.tokenize_events(ev, ty, b.W)
    assert stored_err(to_np(tok).reshape(U, L, d), ref, dtype) <= TOL[dtype]
    cache = ot.Cache(m, U, L)
    ot.onetrans_stage1_encode(m, cache, list(range(U)), tok.view(U, L, d), m.workspace(ot.OP_STAGE1, U, L))
    torch.cuda.synchronize()
    for u in range(U):
        kv = O.stage1(ref[u], b.W, sh.L_NS, sh.n_heads, EPS)   # the oracle's own tokens
        for n, (K, V) in enumerate(kv):
            got = to_np(cache.gather(u, n, L))
            assert stored_err(got[0], K, dtype) <= TOL[dtype] and stored_err(got[1], V, dtype) <= TOL[dtype], (u, n)


@pytest.mark.parametrize("dtype,policy", [("bf16", 0), ("bf16", 1), ("fp32", 0)])
def test_append_small_crosses_page_boundary(dtype, policy):
    ot.onetrans_set_kernel_policy(policy)
    sh = shape(n_layers=2)
    b = build(sh, 104, dtype, event_dim=64)
    U, L_S, dL = 2, 60, 7
    S = gen_normal(9, (U, L_S, sh.d), dtype)
    ev = gen_normal(10, (U, dL, 64), dtype)
    ty = random_types(11, (U, dL), 3)
    m = b.model
    cache = ot.Cache(m, U, 128)
    ot.onetrans_stage1_encode(m, cache, [1, 0], to_dev(S, tdt(dtype)), m.workspace(ot.OP_STAGE1, U, L_S))
    ot.onetrans_cache_append(m, cache, [1, 0], to_dev(ev, tdt(dtype)),
                             torch.from_numpy(ty).cuda(), m.workspace(ot.OP_APPEND, U, dL))
    torch.cuda.synchronize()
    NS = gen_normal(12, (4, sh.L_NS, sh.d), dtype)
    out = torch.empty(4, sh.L_NS, sh.d, dtype=torch.float32, device="cuda")
    ot.onetrans_stage2_score(m, cache, [1, 0], [0, 2, 4], to_dev(NS, tdt(dtype)), out,
                             m.workspace(ot.OP_STAGE2, 4, L_S + dL))
    torch.cuda.synchronize()
    out = to_np(out)
    for u, slot in enumerate([1, 0]):
        assert cache.length(slot) == L_S + dL
        new = O.tokenize_events(ev[u], ty[u], b.W)
        kv = O.append(O.stage1(S[u], b.W, sh.L_NS, sh.n_heads, EPS), new, b.W, sh.n_heads, EPS)
        for n, (K, V) in enumerate(kv):
            got = to_np(cache.gather(slot, n, L_S + dL))
            assert stored_err(got[0], K, dtype) <= TOL[dtype]
            assert stored_err(got[1], V, dtype) <= TOL[dtype]
        for c in range(2 * u, 2 * u + 2):
            r = O.stage2(kv, NS[c], b.W, sh.n_heads, EPS)
            assert rel_err(out[c], r) <= TOL[dtype]


@pytest.mark.parametrize("dtype,policy", [("bf16", 0), ("bf16", 1), ("fp32", 0)])
def test_autosplit_ragged_rows(dtype, policy):
    ot.onetrans_set_kernel_policy(policy)
    sh = shape(n_layers=1)
    b = build(sh, 105, dtype)
    N = 300
    feats = gen_normal(13, (N, sh.ns_feat), dtype)
    ns = torch.empty(N, sh.L_NS, sh.d, dtype=tdt(dtype), device="cuda")
    ot.onetrans_tokenize_autosplit(b.model, to_dev(feats, tdt(dtype)), ns, b.model.workspace(ot.OP_AUTOSPLIT, N))
    torch.cuda.synchronize()
    ref = O.autosplit(feats, b.W, sh.L_NS)
    assert stored_err(to_np(ns), ref, dtype) <= TOL[dtype]


# --------------------------------------------------------- exact checks --

def test_causal_mask_exact_on_gpu():
    """Perturbing NS inputs leaves every S output row bit-identical, and
    perturbing S row t leaves rows < t bit-identical (the kernels are
    deterministic, so any leak of a masked key shows as a bit change)."""
    sh = shape(n_layers=2)
    b = build(sh, 106, "bf16")
    L_S = 150
    X0 = gen_normal(14, (2, L_S + sh.L_NS, sh.d), "bf16")
    base = run_forward(b, X0)
    X1 = X0.copy()
    X1[:, L_S:] = gen_normal(15, (2, sh.L_NS, sh.d), "bf16")
    out1 = run_forward(b, X1)
    np.testing.assert_array_equal(out1[:, :L_S], base[:, :L_S])
    assert np.abs(out1[:, L_S:] - base[:, L_S:]).max() > 0
    X2 = X0.copy()
    X2[:, 97] += 1.0
    out2 = run_forward(b, X2)
    np.testing.assert_array_equal(out2[:, :97], base[:, :97])


def test_schedule_query_and_cache_pages_exact():
    sh = shape(n_layers=6)
    sched = linear_pyramid(1190, 12, 6)
    b = build(sh, 107, "bf16", pyramid=sched)
    assert b.model.schedule(1178) == sched == [1190, 954, 719, 483, 248, 12]
    cache = ot.Cache(b.model, 3, 1178)
    S = gen_normal(16, (2, 1178, sh.d), "bf16")
    ot.onetrans_stage1_encode(b.model, cache, [2, 0], to_dev(S, torch.bfloat16),
                              b.model.workspace(ot.OP_STAGE1, 2, 1178))
    torch.cuda.synchronize()
    s_rows = [1178, 1178, 942, 707, 471, 236]
    max_pages = (1178 + 63) // 64
    table = cache.pool[: 3 * 6 * max_pages * 4].view(torch.int32).cpu().numpy().reshape(3, 6, max_pages)
    seen = set()
    base = cache.pool.data_ptr()
    for slot in (2, 0):
        for n, s in enumerate(s_rows):
            npg = (s + 63) // 64
            pages = table[slot, n, :npg]
            assert (pages >= 0).all() and (table[slot, n, npg:] == -1).all()
            seen.update(pages.tolist())
            for t in (0, s - 1):
                p = cache.row_ptr(slot, n, 1, 3, t) - base
                page = pages[t // 64]
                tb = (3 * 6 * max_pages * 4 + 255) // 256 * 256
                assert p == tb + (page * 2 * sh.d * 64 + ((1 * 4 + 3) * 64 + t % 64) * 64) * 2
    assert len(seen) == 2 * sum((s + 63) // 64 for s in s_rows)


# ------------------------------------------- full-size workloads, sampled --

def test_forward_d384_small():
    """The wider shape (d = 384, 4 heads of 96, FFN 1536, 16 NS tokens) at a
    small size: 384-column GEMM tiles (W^O, QKV of 1152 = 3 x 384, the FFN
    down-projection with the next RMSNorm) and d_h = 96 attention, 3 users x
    (200 + 16) tokens through a 2-layer pyramid."""
    sh = shape(n_layers=2, d=384, dff=1536, L_NS=16)
    L_S = 200
    pyr = linear_pyramid(L_S + sh.L_NS, sh.L_NS, 2)
    b = build(sh, 77, "bf16", pyramid=pyr)
    X0 = gen_normal(78, (3, L_S + sh.L_NS, sh.d), "bf16")
    got = run_forward(b, X0)
    for u in range(3):
        ref = O.forward(X0[u:u + 1], b.W, sh.L_NS, sh.n_heads, EPS, pyr)[0]
        assert rel_err(got[u], ref) <= TOL["bf16"]


def test_stage1_stage2_d384_small():
    """Stage I + II of the wider shape (d_h = 96, 16 NS tokens): the
    two-box head layout in both attention modes, ragged candidate counts
    (a CTA of 8 candidates' 128 NS rows, a partial one and a user with none)."""
    sh = shape(n_layers=2, d=384, dff=1536, L_NS=16)
    L_S = 200
    sched = [L_S + sh.L_NS, sh.L_NS]
    b = build(sh, 91, "bf16", pyramid=sched)
    U = 3
    S = gen_normal(92, (U, L_S, sh.d), "bf16")
    counts = [11, 0, 3]
    offs = np.concatenate([[0], np.cumsum(counts)]).tolist()
    NS = gen_normal(93, (offs[-1], sh.L_NS, sh.d), "bf16")
    cache, out = run_stage12(b, S, NS, offs)
    for u in range(U):
        kv = O.stage1(S[u], b.W, sh.L_NS, sh.n_heads, EPS, sched)
        for n, (K, V) in enumerate(kv):
            got = to_np(cache.gather(u, n, K.shape[0]))
            assert stored_err(got[0], K, "bf16") <= TOL["bf16"]
            assert stored_err(got[1], V, "bf16") <= TOL["bf16"]
        for c in range(offs[u], offs[u + 1]):
            assert rel_err(out[c], O.stage2(kv, NS[c], b.W, sh.n_heads, EPS)) <= TOL["bf16"], (u, c)


def test_zero_work_calls_launch_nothing():
    """Calls with no work return without error and change nothing: no
    features, no samples, no users, users without candidates, no appended
    events (NULL data pointers included)."""
    sh = shape(n_layers=2)
    b = build(sh, 121, "bf16", event_dim=64)
    m = b.model
    bf = torch.bfloat16
    empty_ws = torch.empty(0, dtype=torch.uint8, device="cuda")
    ot.onetrans_tokenize_autosplit(m, torch.empty(0, sh.ns_feat, dtype=bf, device="cuda"),
                                   torch.empty(0, sh.L_NS, sh.d, dtype=bf, device="cuda"), empty_ws)
    ot.onetrans_forward(m, torch.empty(0, 40 + sh.L_NS, sh.d, dtype=bf, device="cuda"),
                        torch.empty(0, 40 + sh.L_NS, sh.d, dtype=torch.float32, device="cuda"), empty_ws)
    U, L_S = 2, 70
    cache = ot.Cache(m, U, L_S + 8)
    ot.onetrans_stage1_encode(m, cache, [], torch.empty(0, L_S, sh.d, dtype=bf, device="cuda"), empty_ws)
    assert cache.length(0) == 0 and cache.length(1) == 0
    S = gen_normal(122, (U, L_S, sh.d), "bf16")
    ot.onetrans_stage1_encode(m, cache, [0, 1], to_dev(S, bf), m.workspace(ot.OP_STAGE1, U, L_S))
    torch.cuda.synchronize()
    before = to_np(cache.gather(1, 0, L_S))
    ot.onetrans_stage2_score(m, cache, [0, 1], [0, 0, 0], torch.empty(0, sh.L_NS, sh.d, dtype=bf, device="cuda"),
                             torch.empty(0, sh.L_NS, sh.d, dtype=torch.float32, device="cuda"), empty_ws)
    ot.onetrans_cache_append(m, cache, [0, 1], torch.empty(U, 0, 64, dtype=bf, device="cuda"),
                             torch.empty(U, 0, dtype=torch.int32, device="cuda"), empty_ws)
    torch.cuda.synchronize()
    assert cache.length(0) == L_S and cache.length(1) == L_S
    np.testing.assert_array_equal(to_np(cache.gather(1, 0, L_S)), before)


def test_long_sequence_beyond_cached_page_ids():
    """8400 cached tokens = 132 pages per layer, past the 128 page ids the
    attention kernel keeps in shared memory: the remaining ids come from the
    page table in global memory, in Stage I's causal attention (100 tail
    queries over up to 8400 keys) and in Stage II."""
    sh = shape(n_layers=2)
    L_S = 8400
    sched = [112, sh.L_NS]
    b = build(sh, 131, "bf16", pyramid=sched)
    S = gen_normal(132, (1, L_S, sh.d), "bf16")
    NS = gen_normal(133, (3, sh.L_NS, sh.d), "bf16")
    cache, out = run_stage12(b, S, NS, [0, 3])
    kv = O.stage1(S[0], b.W, sh.L_NS, sh.n_heads, EPS, sched)
    K0 = to_np(cache.gather(0, 0, L_S))
    assert stored_err(K0[0], kv[0][0], "bf16") <= TOL["bf16"] and stored_err(K0[1], kv[0][1], "bf16") <= TOL["bf16"]
    K1 = to_np(cache.gather(0, 1, kv[1][0].shape[0]))
    assert stored_err(K1[0], kv[1][0], "bf16") <= TOL["bf16"] and stored_err(K1[1], kv[1][1], "bf16") <= TOL["bf16"]
    for c in range(3):
        assert rel_err(out[c], O.stage2(kv, NS[c], b.W, sh.n_heads, EPS)) <= TOL["bf16"]


def _full(name):
    wl = WORKLOADS[name]
    b = build(wl.shape, wl.seed_weights, wl.dtype, pyramid=list(wl.pyramid) if wl.pyramid else None,
              event_dim=wl.event_dim)
    return wl, b


def test_kv_serving_full_size_sampled():
    """The benchmark's workload and launch sequence: auto-split of 16 x 512
    candidates on a second stream beside Stage I of 16 users x 1178, then
    Stage II.  The two-stream runs (repeated, cache rewritten each time) must
    reproduce a one-stream run bit for bit; the oracle checks sampled users
    and candidates of it."""
    wl, b = _full("kv_serving")
    sh, U, C = wl.shape, wl.users, wl.cands
    S = gen_normal(wl.seed_inputs, (U, wl.L_S, sh.d), "bf16")
    feats = gen_normal(wl.seed_inputs + 100, (U * C, sh.ns_feat), "bf16")
    m = b.model
    S_d, F_d = to_dev(S, torch.bfloat16), to_dev(feats, torch.bfloat16)
    ns = torch.empty(U * C, sh.L_NS, sh.d, dtype=torch.bfloat16, device="cuda")
    cache = ot.Cache(m, U, wl.L_S)
    out = torch.empty(U * C, sh.L_NS, sh.d, dtype=torch.float32, device="cuda")
    ws_a = m.workspace(ot.OP_AUTOSPLIT, U * C)
    ws_1 = m.workspace(ot.OP_STAGE1, U, wl.L_S)
    ws_2 = m.workspace(ot.OP_STAGE2, U * C, wl.L_S)
    slots, offs = list(range(U)), [u * C for u in range(U + 1)]

    ot.onetrans_tokenize_autosplit(m, F_d, ns, ws_a)
    ot.onetrans_stage1_encode(m, cache, slots, S_d, ws_1)
    ot.onetrans_stage2_score(m, cache, slots, offs, ns, out, ws_2)
    torch.cuda.synchronize()
    out_seq, ns_seq = out.clone(), ns.clone()

    main, side = torch.cuda.current_stream(), torch.cuda.Stream()
    ev_in, ev_tok = torch.cuda.Event(), torch.cuda.Event()
    for _ in range(3):
        ns.zero_()
        out.zero_()
        ev_in.record(main)
        side.wait_event(ev_in)
        ot.onetrans_tokenize_autosplit(m, F_d, ns, ws_a, stream=side)
        ev_tok.record(side)
        ot.onetrans_stage1_encode(m, cache, slots, S_d, ws_1)
        main.wait_event(ev_tok)
        ot.onetrans_stage2_score(m, cache, slots, offs, ns, out, ws_2)
        torch.cuda.synchronize()
        assert torch.equal(ns, ns_seq) and torch.equal(out, out_seq)

    out, NS = to_np(out_seq), to_np(ns_seq)
    for u in (0, U - 1):
        kv = O.stage1(S[u], b.W, sh.L_NS, sh.n_heads, EPS, wl.pyramid)
        for c in (u * C, u * C + 317, u * C + C - 1):
            ns_ref = O.autosplit(feats[c:c + 1], b.W, sh.L_NS)[0]     # the oracle's own tokens
            assert stored_err(NS[c], ns_ref, "bf16") <= TOL["bf16"]
            r = O.stage2(kv, ns_ref, b.W, sh.n_heads, EPS)
            assert rel_err(out[c], r) <= TOL["bf16"]


def test_kv_serving_pipeline_matches_one_stream():
    """The benchmark's serving pipeline (batch k+1's auto-split and Stage I on
    side streams before batch k's Stage II; two banks of cache and NS
    tokens) reproduces, bit for bit, each batch run alone on one stream."""
    import bench
    wk = bench.KVServing(0)
    m, main, n = wk.model, torch.cuda.current_stream(), 5
    refs = []
    cache = ot.Cache(m, wk.U, wk.wl.L_S)
    ns, out = torch.empty_like(wk.ns[0]), torch.empty_like(wk.out)
    for i in range(n):
        wk.set_inputs(i)
        ot.onetrans_tokenize_autosplit(m, wk.F, ns, wk.ws_a)
        ot.onetrans_stage1_encode(m, cache, wk.slots, wk.S, wk.ws_1)
        ot.onetrans_stage2_score(m, cache, wk.slots, wk.offs, ns, out, wk.ws_2)
        refs.append(out.clone())
    got = []
    for i in range(n):
        wk.set_inputs(i)
        wk.front(i, main)
        if i >= 1:
            wk.back(i - 1, main)
            got.append(wk.out.clone())
    wk.back(n - 1, main)
    got.append(wk.out.clone())
    torch.cuda.synchronize()
    for i in range(n):
        assert torch.equal(got[i], refs[i]), i
    assert not torch.equal(refs[0], refs[1])


def test_append_pipeline_matches_serial():
    """The benchmark's append pipeline (batch k+1's append and auto-split on
    side streams before batch k's Stage II, each batch on its own prepared
    cache) gives, bit for bit, what the same batches give run one after
    another on one stream."""
    import bench
    n = 4
    wk = bench.Append(0, users=16, cands=32)
    main = torch.cuda.current_stream()
    wk.prepare(2 * n)
    # every batch its own candidates and events, so a batch that read another
    # batch's bank or cache would show
    F0, ev0 = wk.F, wk.ev
    Fs = [torch.roll(F0, 37 * i, 0).contiguous() for i in range(n)]
    evs = [torch.roll(ev0, i, 0).contiguous() for i in range(n)]
    serial = []
    for i in range(n):
        wk.F, wk.ev = Fs[i], evs[i]
        wk.front(i, main, serial=True)
        wk.back(i, main)
        serial.append(wk.out.clone())
    got = []
    for i in range(n):
        wk.F, wk.ev = Fs[i], evs[i]
        wk.front(i, main)
        if i >= 1:
            wk.back(i - 1, main)
            got.append(wk.out.clone())
    wk.back(n - 1, main)
    got.append(wk.out.clone())
    torch.cuda.synchronize()
    for i in range(n):
        assert torch.equal(got[i], serial[i]), i
    assert torch.isfinite(serial[0]).all() and not torch.equal(serial[0], serial[1])


def test_s_forward_full_size_sampled():
    wl, b = _full("s_forward")
    sh = wl.shape
    X0 = gen_normal(wl.seed_inputs, (wl.users, wl.L0, sh.d), "bf16")
    got = run_forward(b, X0)
    for u in (0, wl.users - 1):
        ref = O.forward(X0[u:u + 1], b.W, sh.L_NS, sh.n_heads, EPS, wl.pyramid)[0]
        assert rel_err(got[u], ref) <= TOL["bf16"]


def test_append_full_size_sampled():
    wl, b = _full("append")
    sh, U, dL = wl.shape, wl.users, wl.dL
    m = b.model
    S = gen_normal(wl.seed_inputs, (U, wl.L_S, sh.d), "bf16")
    ev = gen_normal(wl.seed_inputs + 200, (U, dL, wl.event_dim), "bf16")
    ty = random_types(wl.seed_inputs + 300, (U, dL), sh.n_types)
    cache = ot.Cache(m, U, wl.L_S + dL)
    ot.onetrans_stage1_encode(m, cache, list(range(U)), to_dev(S, torch.bfloat16),
                              m.workspace(ot.OP_STAGE1, U, wl.L_S))
    ot.onetrans_cache_append(m, cache, list(range(U)), to_dev(ev, torch.bfloat16),
                             torch.from_numpy(ty).cuda(), m.workspace(ot.OP_APPEND, U, dL))
    C = wl.cands
    NS = gen_normal(wl.seed_inputs + 400, (U * C, sh.L_NS, sh.d), "bf16")
    out = torch.empty(U * C, sh.L_NS, sh.d, dtype=torch.float32, device="cuda")
    ot.onetrans_stage2_score(m, cache, list(range(U)), [u * C for u in range(U + 1)],
                             to_dev(NS, torch.bfloat16), out, m.workspace(ot.OP_STAGE2, U * C, wl.L_S + dL))
    torch.cuda.synchronize()
    out = to_np(out)
    u = U - 1
    kv = O.append(O.stage1(S[u], b.W, sh.L_NS, sh.n_heads, EPS),
                  O.tokenize_events(ev[u], ty[u], b.W), b.W, sh.n_heads, EPS)
    got = to_np(cache.gather(u, 5, wl.L_S + dL))
    assert stored_err(got[0], kv[5][0], "bf16") <= TOL["bf16"]
    for c in (u * C, u * C + C - 1):
        assert rel_err(out[c], O.stage2(kv, NS[c], b.W, sh.n_heads, EPS)) <= TOL["bf16"]


def test_l_forward_full_size_sampled():
    wl, b = _full("l_forward")
    sh = wl.shape
    X0 = gen_normal(wl.seed_inputs, (wl.users, wl.L0, sh.d), "bf16")
    got = run_forward(b, X0)
    u = wl.users - 1
    ref = O.forward(X0[u:u + 1], b.W, sh.L_NS, sh.n_heads, EPS, wl.pyramid)[0]
    assert rel_err(got[u], ref) <= TOL["bf16"]
