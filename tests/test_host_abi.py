"""Host-side logic of the C ABI, run without a GPU: symbol exports, argument
and shape validation, schedules, workspace and cache sizing, page-pool
bookkeeping errors.  Device pointers here are fake aligned addresses; every
path exercised returns before any CUDA call."""
import ctypes
import os
import re

import pytest

import unified_transformer_recommender_b200 as ot
from onetrans_synth import linear_pyramid

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "onetrans.h")
FAKE = 0x7f0000000000  # 256-byte aligned stand-in for a device pointer, never dereferenced


def declared_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"ONETRANS_API\s+[\w\s\*]+?\b(onetrans_\w+)\s*\(", txt)))


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) == 28
    for n in names:
        assert hasattr(ot.lib, n), n
    assert set(names) == set(ot.SYMBOLS)
    assert ot.lib.onetrans_version() == 100


class FakeModel:
    """A model handle whose weight pointers are fake device addresses."""

    def __init__(self, n_layers=6, d=256, H=4, dff=1024, L_NS=12, pyramid=None, mode=ot.BF16,
                 page=64, n_beh=0, event_dim=0, F=512, Hh=3072, align=256, null_field=None, head=()):
        self.arrs = []
        self.pyr = (ot.I32 * len(pyramid))(*pyramid) if pyramid else None
        self.cfg = ot.Config(n_layers, d, H, dff, L_NS, F, Hh, n_beh, event_dim,
                             ctypes.cast(self.pyr, ot.PI32) if self.pyr else None, 1e-6, mode, page)
        w = ot.Weights()
        addr = FAKE
        for f in ot._WEIGHT_FIELDS:
            if f == null_field:
                continue
            arr = (ot.P * n_layers)(*[addr + i * align for i in range(n_layers)])
            self.arrs.append(arr)
            setattr(w, f, ctypes.cast(arr, ot.PP))
        for f in ot._TOK_FIELDS:
            setattr(w, f, addr)
        if n_beh:
            for f in ot._BEH_FIELDS:
                arr = (ot.P * n_beh)(*[addr] * n_beh)
                self.arrs.append(arr)
                setattr(w, f, ctypes.cast(arr, ot.PP))
            w.type_emb = addr
        for f, a in zip(ot._HEAD_FIELDS, head):   # (w_head, b_head) addresses, None to leave one out
            setattr(w, f, a)
        self.w = w
        self.h = ot.P()
        self.status = ot.lib.onetrans_model_create(ctypes.byref(self.cfg), ctypes.byref(w), ctypes.byref(self.h))

    def __del__(self):
        if self.h.value:
            ot.lib.onetrans_model_destroy(self.h)


def test_model_create_validation():
    assert FakeModel().status == ot.OK
    assert FakeModel(pyramid=linear_pyramid(1190, 12, 6)).status == ot.OK
    assert FakeModel(H=3).status == ot.ERR_SHAPE                  # d % H
    assert FakeModel(H=32).status == ot.ERR_UNSUPPORTED           # d_h = 8
    assert FakeModel(page=32).status == ot.ERR_UNSUPPORTED
    assert FakeModel(mode=7).status == ot.ERR_INVALID_ARG
    assert FakeModel(null_field="W2_NS").status == ot.ERR_INVALID_ARG
    assert FakeModel(align=8).status == ot.ERR_INVALID_ARG        # misaligned weight
    assert FakeModel(pyramid=[1190, 954, 960, 483, 248, 12]).status == ot.ERR_SHAPE   # increasing
    assert FakeModel(pyramid=[1190, 954, 719, 483, 248, 11]).status == ot.ERR_SHAPE   # below L_NS
    assert FakeModel(n_layers=0).status == ot.ERR_SHAPE
    h = ot.P()
    assert ot.lib.onetrans_model_create(None, None, ctypes.byref(h)) == ot.ERR_INVALID_ARG


def _schedule(fm, L_S):
    out = (ot.I32 * fm.cfg.n_layers)()
    st = ot.lib.onetrans_schedule(fm.h, L_S, out)
    return st, list(out)


def test_schedule_is_exact():
    sched = linear_pyramid(1190, 12, 6)
    fm = FakeModel(pyramid=sched)
    assert _schedule(fm, 1178) == (ot.OK, sched)
    assert _schedule(fm, 1000)[0] == ot.ERR_SHAPE                 # 1190 > L0 = 1012
    fm2 = FakeModel()
    assert _schedule(fm2, 100) == (ot.OK, [112] * 6)
    fm3 = FakeModel(n_layers=8, d=384, L_NS=16, pyramid=linear_pyramid(2064, 16, 8))
    assert _schedule(fm3, 2048) == (ot.OK, [2064, 1771, 1479, 1186, 894, 601, 309, 16])


def _ws(fm, op, n, L):
    out = ot.SZ(0)
    st = ot.lib.onetrans_workspace_size(fm.h, op, n, L, ctypes.byref(out))
    return st, out.value


def test_workspace_sizes_grow_with_work():
    fm = FakeModel(pyramid=linear_pyramid(1190, 12, 6))
    for op, L in ((ot.OP_FORWARD, 1178), (ot.OP_STAGE1, 1178), (ot.OP_STAGE2, 1178), (ot.OP_AUTOSPLIT, 0)):
        st1, a = _ws(fm, op, 16, L)
        st2, b = _ws(fm, op, 64, L)
        assert st1 == st2 == ot.OK and 0 < a < b
    fmA = FakeModel(n_beh=3, event_dim=64)
    st, a = _ws(fmA, ot.OP_APPEND, 256, 16)
    assert st == ot.OK and a > 256 * 16 * 256 * 2 * 8
    # Stage I of 16 x 1178 holds h for all rows plus the tail-row buffers
    st, b1 = _ws(fm, ot.OP_STAGE1, 16, 1178)
    assert b1 >= 16 * 1178 * 256 * 2 * 8
    assert _ws(fm, 9, 1, 1)[0] == ot.ERR_INVALID_ARG
    assert _ws(fm, ot.OP_FORWARD, -1, 1)[0] == ot.ERR_SHAPE


def _cache(fm, n_slots, max_L, pool=FAKE, size=None):
    sz = ot.SZ(0)
    assert ot.lib.onetrans_cache_size(fm.h, n_slots, max_L, ctypes.byref(sz)) == ot.OK
    h = ot.P()
    st = ot.lib.onetrans_cache_init(fm.h, pool, sz.value if size is None else size, n_slots, max_L, ctypes.byref(h))
    return st, sz.value, h


def test_cache_size_formula_and_init_errors():
    sched = linear_pyramid(1190, 12, 6)
    fm = FakeModel(pyramid=sched)
    st, size, h = _cache(fm, 16, 1178)
    assert st == ot.OK
    s_rows = [1178, 1178, 942, 707, 471, 236]
    pages = 16 * sum((s + 63) // 64 for s in s_rows)
    table = (16 * 6 * 19 * 4 + 255) // 256 * 256
    assert size == table + pages * (2 * 256 * 64 * 2)
    ot.lib.onetrans_cache_destroy(h)
    assert _cache(fm, 16, 1178, size=size - 1)[0] == ot.ERR_CAPACITY
    assert _cache(fm, 16, 1178, pool=FAKE + 16)[0] == ot.ERR_INVALID_ARG
    ln = ot.I32(0)
    st, _, h = _cache(fm, 2, 100)
    assert ot.lib.onetrans_cache_length(h, 1, ctypes.byref(ln)) == ot.OK and ln.value == 0
    assert ot.lib.onetrans_cache_length(h, 2, ctypes.byref(ln)) == ot.ERR_SHAPE
    ot.lib.onetrans_cache_destroy(h)


def test_entry_point_argument_errors_before_any_launch():
    sched = linear_pyramid(1190, 12, 6)
    fm = FakeModel(pyramid=sched, n_beh=3, event_dim=64)
    st, size, c = _cache(fm, 4, 1178)
    assert st == ot.OK
    ws, big = FAKE, 1 << 40
    slots = (ot.I32 * 2)(0, 1)
    dup = (ot.I32 * 2)(1, 1)
    bad = (ot.I32 * 2)(0, 4)
    # append is defined for non-pyramid stacks only
    assert ot.lib.onetrans_cache_append(fm.h, c, slots, 2, FAKE, FAKE, 16, ws, big, None) == ot.ERR_UNSUPPORTED
    # slot validation
    assert ot.lib.onetrans_stage1_encode(fm.h, c, dup, 2, FAKE, 1178, ws, big, None) == ot.ERR_INVALID_ARG
    assert ot.lib.onetrans_stage1_encode(fm.h, c, bad, 2, FAKE, 1178, ws, big, None) == ot.ERR_SHAPE
    # sequence longer than the cache was sized for
    assert ot.lib.onetrans_stage1_encode(fm.h, c, slots, 2, FAKE, 1179, ws, big, None) in (ot.ERR_CAPACITY, ot.ERR_SHAPE)
    # workspace too small
    assert ot.lib.onetrans_stage1_encode(fm.h, c, slots, 2, FAKE, 1178, ws, 1024, None) == ot.ERR_CAPACITY
    # schedule does not fit the sequence
    assert ot.lib.onetrans_stage1_encode(fm.h, c, slots, 2, FAKE, 500, ws, big, None) == ot.ERR_SHAPE
    # Stage II on empty slots / bad CSR
    offs = (ot.I32 * 3)(0, 5, 9)
    assert ot.lib.onetrans_stage2_score(fm.h, c, slots, 2, offs, FAKE, FAKE, None, ws, big, None) == ot.ERR_SHAPE
    offs_bad = (ot.I32 * 3)(0, 5, 3)
    assert ot.lib.onetrans_stage2_score(fm.h, c, slots, 2, offs_bad, FAKE, FAKE, None, ws, big, None) == ot.ERR_SHAPE
    # logits asked of a model without the scoring head
    assert ot.lib.onetrans_stage2_score(fm.h, c, slots, 2, offs, FAKE, FAKE, FAKE, ws, big, None) == ot.ERR_UNSUPPORTED
    # misaligned workspace / inputs
    assert ot.lib.onetrans_forward(fm.h, FAKE, 2, 1178, FAKE, FAKE + 16, big, None) == ot.ERR_INVALID_ARG
    assert ot.lib.onetrans_forward(fm.h, FAKE + 2, 2, 1178, FAKE, ws, big, None) == ot.ERR_INVALID_ARG
    assert ot.lib.onetrans_forward(fm.h, FAKE, 2, 1178, FAKE, ws, 1024, None) == ot.ERR_CAPACITY
    assert ot.lib.onetrans_forward(fm.h, FAKE, 2, 900, FAKE, ws, big, None) == ot.ERR_SHAPE
    ot.lib.onetrans_cache_destroy(c)
    # a cache belongs to the model it was made for
    fm2 = FakeModel(pyramid=sched)
    st, _, c2 = _cache(fm2, 4, 1178)
    assert ot.lib.onetrans_stage1_encode(fm.h, c2, slots, 2, FAKE, 1178, ws, big, None) == ot.ERR_INVALID_ARG
    ot.lib.onetrans_cache_destroy(c2)


def test_tokenize_events_argument_errors_before_any_launch():
    fm = FakeModel(n_beh=3, event_dim=64)
    assert fm.status == ot.OK
    # no events: nothing to do, the data pointers may be NULL
    assert ot.lib.onetrans_tokenize_events(fm.h, None, None, 0, None, None) == ot.OK
    assert ot.lib.onetrans_tokenize_events(fm.h, FAKE, FAKE, -1, FAKE, None) == ot.ERR_SHAPE
    assert ot.lib.onetrans_tokenize_events(fm.h, FAKE + 2, FAKE, 8, FAKE, None) == ot.ERR_INVALID_ARG
    assert ot.lib.onetrans_tokenize_events(fm.h, FAKE, FAKE, 8, FAKE + 8, None) == ot.ERR_INVALID_ARG
    assert ot.lib.onetrans_tokenize_events(fm.h, FAKE, None, 8, FAKE, None) == ot.ERR_INVALID_ARG
    assert ot.lib.onetrans_tokenize_events(None, FAKE, FAKE, 8, FAKE, None) == ot.ERR_INVALID_ARG
    # a model without behavior MLPs has no event tokenizer
    fm0 = FakeModel()
    assert ot.lib.onetrans_tokenize_events(fm0.h, FAKE, FAKE, 8, FAKE, None) == ot.ERR_UNSUPPORTED


def test_merge_intent_order_argument_errors_before_any_launch():
    fm = FakeModel(n_beh=3, event_dim=64)
    assert fm.status == ot.OK

    def merge(m, events, lens, types, sep, tokens, n=None):
        n = len(lens) if n is None else n
        L = (ot.I64 * max(len(lens), 1))(*lens)
        T = (ot.I32 * max(len(types), 1))(*types)
        return ot.lib.onetrans_merge_intent_order(m, events, L, T, n, sep, tokens, None)

    # one empty sequence: no rows at all, nothing launched, pointers may be NULL
    assert merge(fm.h, None, [0], [1], None, None) == ot.OK
    assert merge(fm.h, FAKE, [4, 3], [0, 1], FAKE, FAKE, n=0) == ot.ERR_SHAPE
    assert merge(fm.h, FAKE, [1] * 9, [0] * 9, FAKE, FAKE) == ot.ERR_UNSUPPORTED   # above 8 sequences
    assert merge(fm.h, FAKE, [4, -1], [0, 1], FAKE, FAKE) == ot.ERR_SHAPE
    assert merge(fm.h, FAKE, [4, 3], [0, 3], FAKE, FAKE) == ot.ERR_INVALID_ARG     # behavior id out of range
    assert merge(fm.h, FAKE, [4, 3], [0, -1], FAKE, FAKE) == ot.ERR_INVALID_ARG
    assert merge(fm.h, FAKE, [4, 3], [0, 1], None, FAKE) == ot.ERR_INVALID_ARG     # two sequences need [SEP]
    assert merge(fm.h, FAKE + 2, [4, 3], [0, 1], FAKE, FAKE) == ot.ERR_INVALID_ARG
    assert merge(fm.h, FAKE, [4, 3], [0, 1], FAKE, FAKE + 8) == ot.ERR_INVALID_ARG
    assert merge(fm.h, None, [4], [0], None, FAKE) == ot.ERR_INVALID_ARG           # events missing
    assert merge(fm.h, FAKE, [2 ** 31], [0], None, FAKE) == ot.ERR_SHAPE
    assert ot.lib.onetrans_merge_intent_order(fm.h, FAKE, None, None, 2, FAKE, FAKE, None) == ot.ERR_INVALID_ARG
    assert merge(None, FAKE, [4, 3], [0, 1], FAKE, FAKE) == ot.ERR_INVALID_ARG
    fm0 = FakeModel()
    assert merge(fm0.h, FAKE, [4, 3], [0, 1], FAKE, FAKE) == ot.ERR_UNSUPPORTED


def test_tokenize_groupwise_argument_errors_and_workspace_before_any_launch():
    fm = FakeModel()
    assert fm.status == ot.OK
    G = fm.cfg.L_NS
    gw = ot.lib.onetrans_tokenize_groupwise
    ws = ctypes.c_void_p(FAKE)
    big = 1 << 40
    args = dict(feats=FAKE, N=8, G=G, F=24, h=40, W1=FAKE, b1=FAKE, W2=FAKE, b2=FAKE, tok=FAKE, ws=ws, n=big)

    def call(m=None, **kw):
        a = dict(args, **kw)
        return gw(fm.h if m is None else m, a["feats"], a["N"], a["G"], a["F"], a["h"], a["W1"], a["b1"],
                  a["W2"], a["b2"], a["tok"], a["ws"], a["n"], None)

    assert call(N=0, feats=None, W1=None, tok=None, ws=None) == ot.OK   # no rows: nothing launched
    assert call(N=-1) == ot.ERR_SHAPE
    assert call(G=G + 1) == ot.ERR_SHAPE                               # one token per group: G = L_NS
    assert call(F=0) == ot.ERR_SHAPE
    assert call(h=0) == ot.ERR_SHAPE
    for k in ("feats", "W1", "b1", "W2", "b2", "tok"):
        assert call(**{k: None}) == ot.ERR_INVALID_ARG, k
    assert call(feats=FAKE + 2) == ot.ERR_INVALID_ARG
    assert call(W2=FAKE + 8) == ot.ERR_INVALID_ARG
    assert call(ws=None) == ot.ERR_INVALID_ARG
    assert call(n=1024) == ot.ERR_CAPACITY                              # hidden layer does not fit
    assert call(m=ctypes.c_void_p(0)) == ot.ERR_INVALID_ARG
    # workspace: the [N, G, h_max] hidden layer in the mode's element type
    out = ot.SZ(0)
    assert ot.lib.onetrans_workspace_size(fm.h, ot.OP_GROUPWISE, 100, 40, ctypes.byref(out)) == ot.OK
    assert out.value == 100 * G * 40 * 2
    assert ot.lib.onetrans_workspace_size(fm.h, ot.OP_GROUPWISE, 100, 0, ctypes.byref(out)) == ot.ERR_SHAPE


def test_stage1_ragged_checks_every_run_before_any_launch():
    """Without a GPU any launch fails with a CUDA error: a call whose first run
    is valid and whose second is not must return the second run's error and
    leave every slot as it was."""
    sched = linear_pyramid(1190, 12, 6)
    fm = FakeModel(pyramid=sched)
    st, size, c = _cache(fm, 4, 1178)
    assert st == ot.OK
    ws, big = FAKE, 1 << 40
    enc = ot.lib.onetrans_stage1_encode_ragged

    def call(slots, lens, ws_bytes=big, s_tok=FAKE, lens_ptr=True):
        S = (ot.I32 * len(slots))(*slots)
        Lp = (ot.I32 * len(lens))(*lens) if lens_ptr else None
        return enc(fm.h, c, S, len(slots), s_tok, Lp, ws, ws_bytes, None)

    assert enc(fm.h, c, None, 0, None, None, None, 0, None) == ot.OK      # no users: nothing launched
    assert call([0, 1], [1178, 1178], lens_ptr=False) == ot.ERR_INVALID_ARG
    assert call([0, 1], [1178, 0]) == ot.ERR_SHAPE
    assert call([0, 0], [1178, 1178]) == ot.ERR_INVALID_ARG              # a slot twice
    assert call([0, 1], [1178, 500]) == ot.ERR_SHAPE                     # second run: schedule does not fit
    assert call([0, 1], [1178, 1179]) == ot.ERR_CAPACITY                 # second run: longer than the pool's rows
    assert call([0, 1], [1178, 1100], ws_bytes=1024) == ot.ERR_CAPACITY  # workspace
    assert call([0, 1], [1178, 1100], s_tok=FAKE + 2) == ot.ERR_INVALID_ARG
    ln = ot.I32(-1)
    for slot in range(4):
        assert ot.lib.onetrans_cache_length(c, slot, ctypes.byref(ln)) == ot.OK and ln.value == 0
    ot.lib.onetrans_cache_destroy(c)


def test_policy_and_status_strings():
    assert ot.lib.onetrans_selftest_bounded_wait(0, None) == ot.ERR_INVALID_ARG
    assert ot.lib.onetrans_selftest_bounded_wait((1 << 20) + 1, None) == ot.ERR_INVALID_ARG
    assert ot.lib.onetrans_set_kernel_policy(2) == ot.ERR_INVALID_ARG
    assert ot.lib.onetrans_set_kernel_policy(0) == ot.OK
    assert ot.status_string(ot.ERR_CAPACITY) == "capacity exceeded"
    assert ot.status_string(123) == "unknown status"


def test_model_left_alive_until_interpreter_exit_is_destroyed_cleanly(tmp_path):
    """A model still referenced by a module global when the interpreter exits
    is collected after the binding's module globals are cleared; its
    destructor must still reach the library.  The weights are host tensors:
    model creation only validates and records their addresses."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    script = tmp_path / "leave_alive.py"
    script.write_text(
        "import sys\n"
        f"sys.path.insert(0, {root!r})\n"
        "import unified_transformer_recommender_b200 as ot\n"
        "from onetrans_synth import ModelShape, make_weights\n"
        "sh = ModelShape(n_layers=2, d=256, n_heads=4, d_ff=1024, L_NS=2, ns_feat=16,\n"
        "                ns_hidden=512, behavior_dims=(8,))\n"
        "MODEL = ot.model_from_arrays(sh, make_weights(sh, 1, 'bf16'), device='cpu')\n"
        "print('made', bool(MODEL.handle.value))\n")
    r = subprocess.run([sys.executable, str(script)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert "made True" in r.stdout
    assert "Exception ignored" not in r.stderr, r.stderr


def test_scoring_head_weights_come_in_pairs():
    assert FakeModel(head=(FAKE, FAKE + 256)).status == ot.OK
    assert FakeModel(head=(FAKE, None)).status == ot.ERR_INVALID_ARG
    assert FakeModel(head=(None, FAKE)).status == ot.ERR_INVALID_ARG
    assert FakeModel(head=(FAKE + 4, FAKE)).status == ot.ERR_INVALID_ARG     # w_head not 16-byte aligned


def test_forward_backward_argument_errors_before_any_launch():
    sched = linear_pyramid(1190, 12, 6)
    fm = FakeModel(pyramid=sched)
    g = ot.Grads()
    arrs = []
    for f in ot._WEIGHT_FIELDS:
        arr = (ot.P * 6)(*[FAKE + i * 256 for i in range(6)])
        arrs.append(arr)
        setattr(g, f, ctypes.cast(arr, ot.PP))
    fb = ot.lib.onetrans_forward_backward
    big = 1 << 40
    assert fb(fm.h, FAKE, 2, 1178, FAKE, FAKE, FAKE, None, FAKE, big, None) == ot.ERR_INVALID_ARG   # no grads
    assert fb(fm.h, None, 0, 1178, None, None, None, ctypes.byref(g), None, 0, None) == ot.OK   # no samples
    assert fb(fm.h, FAKE, 2, 900, FAKE, FAKE, FAKE, ctypes.byref(g), FAKE, big, None) == ot.ERR_SHAPE  # schedule
    assert fb(fm.h, FAKE + 2, 2, 1178, FAKE, FAKE, FAKE, ctypes.byref(g), FAKE, big, None) == ot.ERR_INVALID_ARG
    assert fb(fm.h, FAKE, 2, 1178, FAKE, FAKE, None, ctypes.byref(g), FAKE, big, None) == ot.ERR_INVALID_ARG
    assert fb(fm.h, FAKE, 2, 1178, FAKE, FAKE, FAKE, ctypes.byref(g), FAKE, 1024, None) == ot.ERR_CAPACITY
    arrs[4][3] = FAKE + 4                                              # Wo gradient of layer 3 misaligned
    assert fb(fm.h, FAKE, 2, 1178, FAKE, FAKE, FAKE, ctypes.byref(g), FAKE, big, None) == ot.ERR_INVALID_ARG
    out = ot.SZ(0)
    assert ot.lib.onetrans_workspace_size(fm.h, ot.OP_TRAIN, 2, 1178, ctypes.byref(out)) == ot.OK
    # at least what the forward keeps: the float32 inputs of layers 1..5 and
    # every layer's bf16 attention output and float32 log-sum-exp
    kept = sum(2 * sched[n - 1] * 256 * 4 for n in range(1, 6))
    kept += sum(2 * q * 256 * 2 + 2 * 4 * q * 4 for q in sched)
    assert out.value > kept
