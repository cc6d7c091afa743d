"""Python binding of the OneTrans B200 library (ctypes over include/onetrans.h).

Argument marshalling only: every step of the path runs in the CUDA library
`libonetrans.so` built in this directory.  PyTorch supplies device memory and
streams.  Importing this package loads the library and raises if it is
missing; there is no other implementation behind these calls.

The functions carry the C names (onetrans_forward, onetrans_stage1_encode,
...).  `Model` and `Cache` own the C handles and the pointer tables.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libonetrans.so")

OK, ERR_INVALID_ARG, ERR_SHAPE, ERR_UNSUPPORTED, ERR_CAPACITY, ERR_CUDA, ERR_DEVICE_CHECK = 0, -1, -2, -3, -4, -5, -6
BF16, FP32 = 0, 1
OP_FORWARD, OP_STAGE1, OP_STAGE2, OP_APPEND, OP_AUTOSPLIT, OP_GROUPWISE, OP_TRAIN = 0, 1, 2, 3, 4, 5, 6

SYMBOLS = (
    "onetrans_model_create", "onetrans_model_destroy", "onetrans_workspace_size",
    "onetrans_schedule", "onetrans_cache_size", "onetrans_cache_init",
    "onetrans_cache_destroy", "onetrans_cache_length", "onetrans_cache_row_ptr",
    "onetrans_tokenize_autosplit", "onetrans_stage1_encode", "onetrans_stage1_encode_ragged",
    "onetrans_stage2_score",
    "onetrans_cache_append", "onetrans_forward", "onetrans_set_kernel_policy",
    "onetrans_device_status", "onetrans_status_string", "onetrans_version",
    "onetrans_profile_enable", "onetrans_profile_kinds", "onetrans_profile_read",
    "onetrans_tokenize_autosplit_static", "onetrans_tokenize_events", "onetrans_merge_intent_order",
    "onetrans_tokenize_groupwise", "onetrans_selftest_bounded_wait", "onetrans_forward_backward",
)


class OneTransError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status} ({status_string(status)})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python unified_transformer_recommender_b200/build.py`")
    return ctypes.CDLL(LIB_PATH)


lib = _load()

P = ctypes.c_void_p
I32 = ctypes.c_int32
I64 = ctypes.c_int64
SZ = ctypes.c_size_t
PP = ctypes.POINTER(ctypes.c_void_p)
PI32 = ctypes.POINTER(ctypes.c_int32)
PI64 = ctypes.POINTER(ctypes.c_int64)


class Config(ctypes.Structure):
    _fields_ = [("n_layers", I32), ("d_model", I32), ("n_heads", I32), ("d_ff", I32),
                ("L_NS", I32), ("ns_feat_dim", I32), ("ns_hidden", I32),
                ("n_behaviors", I32), ("event_dim", I32), ("pyramid_q", PI32),
                ("rms_eps", ctypes.c_float), ("mode", I32), ("page_tokens", I32)]


_WEIGHT_FIELDS = ("g_attn", "g_ffn", "Wqkv_S", "Wqkv_NS", "Wo", "W1_S", "b1_S", "W2_S",
                  "b2_S", "W1_NS", "b1_NS", "W2_NS", "b2_NS")
_TOK_FIELDS = ("Wa1", "ba1", "Wa2", "ba2")
_HEAD_FIELDS = ("w_head", "b_head")
_BEH_FIELDS = ("Wb1", "bb1", "Wb2", "bb2")


class Weights(ctypes.Structure):
    _fields_ = ([(f, PP) for f in _WEIGHT_FIELDS] + [(f, P) for f in _TOK_FIELDS]
                + [(f, PP) for f in _BEH_FIELDS] + [("type_emb", P)] + [(f, P) for f in _HEAD_FIELDS])


class Grads(ctypes.Structure):
    """onetrans_grads: per-layer host arrays of float32 device pointers."""
    _fields_ = [(f, PP) for f in _WEIGHT_FIELDS]


def _sig(name, res, *args):
    fn = getattr(lib, name)
    fn.restype = res
    fn.argtypes = list(args)
    return fn


_sig("onetrans_model_create", I32, ctypes.POINTER(Config), ctypes.POINTER(Weights), ctypes.POINTER(P))
_sig("onetrans_model_destroy", I32, P)
_sig("onetrans_workspace_size", I32, P, I32, I64, I32, ctypes.POINTER(SZ))
_sig("onetrans_schedule", I32, P, I32, PI32)
_sig("onetrans_cache_size", I32, P, I32, I32, ctypes.POINTER(SZ))
_sig("onetrans_cache_init", I32, P, P, SZ, I32, I32, ctypes.POINTER(P))
_sig("onetrans_cache_destroy", I32, P)
_sig("onetrans_cache_length", I32, P, I32, PI32)
_sig("onetrans_cache_row_ptr", I32, P, I32, I32, I32, I32, I32, ctypes.POINTER(P))
_sig("onetrans_tokenize_autosplit", I32, P, P, I64, P, P, SZ, P)
_sig("onetrans_tokenize_autosplit_static", I32, P, P, I64, P, P)
_sig("onetrans_stage1_encode", I32, P, P, PI32, I32, P, I32, P, SZ, P)
_sig("onetrans_stage1_encode_ragged", I32, P, P, PI32, I32, P, PI32, P, SZ, P)
_sig("onetrans_stage2_score", I32, P, P, PI32, I32, PI32, P, P, P, P, SZ, P)
_sig("onetrans_cache_append", I32, P, P, PI32, I32, P, P, I32, P, SZ, P)
_sig("onetrans_tokenize_events", I32, P, P, P, I64, P, P)
_sig("onetrans_merge_intent_order", I32, P, P, PI64, PI32, I32, P, P, P)
_sig("onetrans_tokenize_groupwise", I32, P, P, I64, I32, I32, I32, P, P, P, P, P, P, SZ, P)
_sig("onetrans_forward", I32, P, P, I32, I32, P, P, SZ, P)
_sig("onetrans_forward_backward", I32, P, P, I32, I32, P, P, P, P, P, SZ, P)
_sig("onetrans_set_kernel_policy", I32, I32)
_sig("onetrans_device_status", I32, P, PI32)
_sig("onetrans_selftest_bounded_wait", I32, I32, P)
_sig("onetrans_status_string", ctypes.c_char_p, I32)
_sig("onetrans_version", I32)
_sig("onetrans_profile_enable", I32, I32)
_sig("onetrans_profile_kinds", I32)
_sig("onetrans_profile_read", I32, I32, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(I64),
     ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double))


def status_string(s: int) -> str:
    return lib.onetrans_status_string(int(s)).decode()


def _check(fn: str, s: int) -> None:
    if s != OK:
        raise OneTransError(fn, s)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream: Optional[torch.cuda.Stream]) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _i32(vals: Sequence[int]):
    arr = (I32 * len(vals))(*[int(v) for v in vals])
    return arr


def onetrans_set_kernel_policy(policy: int) -> None:
    _check("onetrans_set_kernel_policy", lib.onetrans_set_kernel_policy(int(policy)))


def onetrans_device_status(stream=None) -> int:
    """Reads and clears the device status word: 0, or the failed check's code."""
    code = I32(0)
    s = lib.onetrans_device_status(_stream(stream), ctypes.byref(code))
    if s != ERR_DEVICE_CHECK:
        _check("onetrans_device_status", s)
    return code.value


def onetrans_selftest_bounded_wait(spin_limit: int, stream=None) -> None:
    _check("onetrans_selftest_bounded_wait", lib.onetrans_selftest_bounded_wait(int(spin_limit), _stream(stream)))


def onetrans_profile_enable(on: bool) -> None:
    _check("onetrans_profile_enable", lib.onetrans_profile_enable(1 if on else 0))


def onetrans_profile_read() -> dict:
    """{kernel kind: {launches, ms, flops, bytes}} of the launches recorded
    since profiling was enabled (kinds with no launch omitted)."""
    out = {}
    for k in range(lib.onetrans_profile_kinds()):
        name, n = ctypes.c_char_p(), I64(0)
        ms, fl, by = ctypes.c_double(0), ctypes.c_double(0), ctypes.c_double(0)
        _check("onetrans_profile_read", lib.onetrans_profile_read(k, ctypes.byref(name), ctypes.byref(n),
                                                                   ctypes.byref(ms), ctypes.byref(fl), ctypes.byref(by)))
        if n.value:
            out[name.value.decode()] = {"launches": n.value, "ms": ms.value, "flops": fl.value, "bytes": by.value}
    return out


class Model:
    """Owns an onetrans_model handle.  `weights` maps the header's field names
    to device tensors (per-layer fields: lists of tensors).  The tensors are
    kept referenced for the model's lifetime."""

    def __init__(self, *, n_layers, d_model, n_heads, d_ff, L_NS, weights: Dict,
                 pyramid_q: Optional[Sequence[int]] = None, mode: int = BF16,
                 ns_feat_dim: int = 0, ns_hidden: int = 0, n_behaviors: int = 0,
                 event_dim: int = 0, rms_eps: float = 1e-6, page_tokens: int = 64):
        self._keep = []
        self.dtype = torch.bfloat16 if mode == BF16 else torch.float32
        self._pyr = _i32(pyramid_q) if pyramid_q is not None else None
        self.cfg = Config(n_layers, d_model, n_heads, d_ff, L_NS, ns_feat_dim, ns_hidden,
                          n_behaviors, event_dim,
                          ctypes.cast(self._pyr, PI32) if self._pyr is not None else None,
                          rms_eps, mode, page_tokens)
        w = Weights()
        for f in _WEIGHT_FIELDS + _BEH_FIELDS:
            ts = weights.get(f)
            if ts is None:
                continue
            arr = (P * len(ts))(*[_ptr(self._own(t)) for t in ts])
            self._keep.append(arr)
            setattr(w, f, ctypes.cast(arr, PP))
        for f in _TOK_FIELDS + ("type_emb",) + _HEAD_FIELDS:
            t = weights.get(f)
            if t is not None:
                setattr(w, f, _ptr(self._own(t)))
        self._w = w
        h = P()
        _check("onetrans_model_create", lib.onetrans_model_create(ctypes.byref(self.cfg), ctypes.byref(w), ctypes.byref(h)))
        self.handle = h
        # held by the object so that a model collected at interpreter exit,
        # after the module's globals are cleared, can still be destroyed
        self._destroy = lib.onetrans_model_destroy
        self.n_layers, self.d, self.L_NS = n_layers, d_model, L_NS

    def _own(self, t: torch.Tensor) -> torch.Tensor:
        if t.dtype != self.dtype or not t.is_contiguous():
            raise ValueError("weights must be contiguous tensors of the model dtype")
        self._keep.append(t)
        return t

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and h.value:
            self._destroy(h)
            self.handle = None

    def workspace_size(self, op: int, n: int, L: int = 0) -> int:
        out = SZ(0)
        _check("onetrans_workspace_size", lib.onetrans_workspace_size(self.handle, op, n, L, ctypes.byref(out)))
        return out.value

    def workspace(self, op: int, n: int, L: int = 0, device="cuda") -> torch.Tensor:
        return torch.empty(max(self.workspace_size(op, n, L), 256), dtype=torch.uint8, device=device)

    def schedule(self, L_S: int):
        out = (I32 * self.n_layers)()
        _check("onetrans_schedule", lib.onetrans_schedule(self.handle, L_S, out))
        return list(out)


class Cache:
    """Owns an onetrans_cache handle over a caller-allocated device pool."""

    def __init__(self, model: Model, n_slots: int, max_L_S: int, device="cuda"):
        size = SZ(0)
        _check("onetrans_cache_size", lib.onetrans_cache_size(model.handle, n_slots, max_L_S, ctypes.byref(size)))
        self.pool = torch.empty(size.value, dtype=torch.uint8, device=device)
        h = P()
        _check("onetrans_cache_init", lib.onetrans_cache_init(model.handle, self.pool.data_ptr(), size.value,
                                                                n_slots, max_L_S, ctypes.byref(h)))
        self.handle, self.model = h, model
        self._destroy = lib.onetrans_cache_destroy

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and h.value:
            self._destroy(h)
            self.handle = None

    def length(self, slot: int) -> int:
        out = I32(0)
        _check("onetrans_cache_length", lib.onetrans_cache_length(self.handle, slot, ctypes.byref(out)))
        return out.value

    def row_ptr(self, slot, layer, kind, head, token) -> int:
        out = P()
        _check("onetrans_cache_row_ptr", lib.onetrans_cache_row_ptr(self.handle, slot, layer, kind, head, token,
                                                                      ctypes.byref(out)))
        return out.value

    def gather(self, slot: int, layer: int, length: int) -> torch.Tensor:
        """Cached [2, length, d] K/V rows of (slot, layer), heads concatenated,
        read back page by page (device copies)."""
        m = self.model
        H = m.cfg.n_heads
        dh = m.d // H
        es = 2 if m.dtype == torch.bfloat16 else 4
        out = torch.empty(2, length, m.d, dtype=m.dtype, device=self.pool.device)
        base = self.pool.data_ptr()
        for kind in range(2):
            for h in range(H):
                for t0 in range(0, length, m.cfg.page_tokens):
                    n = min(m.cfg.page_tokens, length - t0)
                    off = self.row_ptr(slot, layer, kind, h, t0) - base
                    src = self.pool[off: off + n * dh * es].view(m.dtype).view(n, dh)
                    out[kind, t0:t0 + n, h * dh:(h + 1) * dh] = src
        return out


# ------------------------------------------------------------- entry points

def onetrans_tokenize_autosplit(model: Model, feats: torch.Tensor, ns_tokens: torch.Tensor,
                                ws: torch.Tensor, stream=None) -> None:
    _check("onetrans_tokenize_autosplit", lib.onetrans_tokenize_autosplit(
        model.handle, _ptr(feats), feats.shape[0], _ptr(ns_tokens), _ptr(ws), ws.numel(), _stream(stream)))


def onetrans_tokenize_autosplit_static(model: Model, feats: torch.Tensor, ns_tokens: torch.Tensor,
                                       stream=None) -> None:
    """Auto-split without a workspace (scratch in the library's fixed array)."""
    _check("onetrans_tokenize_autosplit_static", lib.onetrans_tokenize_autosplit_static(
        model.handle, _ptr(feats), feats.shape[0], _ptr(ns_tokens), _stream(stream)))


def onetrans_tokenize_events(model: Model, events: torch.Tensor, types: torch.Tensor, tokens: torch.Tensor,
                             stream=None) -> None:
    """events [R, event_dim], types [R] int32 (device), tokens [R, d]."""
    _check("onetrans_tokenize_events", lib.onetrans_tokenize_events(
        model.handle, _ptr(events), _ptr(types), events.shape[0], _ptr(tokens), _stream(stream)))


def onetrans_merge_intent_order(model: Model, events: torch.Tensor, seq_len: Sequence[int],
                                seq_type: Sequence[int], sep: Optional[torch.Tensor], tokens: torch.Tensor,
                                stream=None) -> None:
    """events [sum(seq_len), event_dim] (device), the sequences back to back in
    intent order; seq_len / seq_type per sequence (host); sep [d] (device);
    tokens [sum(seq_len) + len(seq_len) - 1, d]."""
    n = len(seq_len)
    lens = (I64 * max(n, 1))(*[int(v) for v in seq_len])
    _check("onetrans_merge_intent_order", lib.onetrans_merge_intent_order(
        model.handle, _ptr(events), lens, _i32(list(seq_type) or [0]), n, _ptr(sep), _ptr(tokens),
        _stream(stream)))


def onetrans_tokenize_groupwise(model: Model, feats: torch.Tensor, W1: torch.Tensor, b1: torch.Tensor,
                                W2: torch.Tensor, b2: torch.Tensor, ns_tokens: torch.Tensor, ws: torch.Tensor,
                                stream=None) -> None:
    """feats [N, G, F_max]; W1 [G, h_max, F_max], b1 [G, h_max], W2 [G, d, h_max],
    b2 [G, d] (zero-padded per group); ns_tokens [N, G, d]."""
    N, G, F_max = feats.shape
    _check("onetrans_tokenize_groupwise", lib.onetrans_tokenize_groupwise(
        model.handle, _ptr(feats), N, G, F_max, W1.shape[1], _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2),
        _ptr(ns_tokens), _ptr(ws), ws.numel(), _stream(stream)))


def onetrans_stage1_encode(model: Model, cache: Cache, slots: Sequence[int], s_tokens: torch.Tensor,
                           ws: torch.Tensor, stream=None) -> None:
    sl = _i32(slots)
    _check("onetrans_stage1_encode", lib.onetrans_stage1_encode(
        model.handle, cache.handle, sl, len(slots), _ptr(s_tokens), s_tokens.shape[1], _ptr(ws), ws.numel(),
        _stream(stream)))


def onetrans_stage1_encode_ragged(model: Model, cache: Cache, slots: Sequence[int], lens: Sequence[int],
                                  s_tokens: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    """s_tokens [sum(lens), d]: user u's lens[u] rows back to back, in the order of slots."""
    _check("onetrans_stage1_encode_ragged", lib.onetrans_stage1_encode_ragged(
        model.handle, cache.handle, _i32(slots), len(slots), _ptr(s_tokens), _i32(list(lens) or [0]), _ptr(ws),
        ws.numel(), _stream(stream)))


def onetrans_stage2_score(model: Model, cache: Cache, slots: Sequence[int], cand_offsets: Sequence[int],
                          ns_tokens: torch.Tensor, ns_out: torch.Tensor, ws: torch.Tensor, stream=None,
                          logits: Optional[torch.Tensor] = None) -> None:
    """ns_tokens [C, L_NS, d]; ns_out [C, L_NS, d] float32; logits [C] float32
    or None (needs the model's w_head / b_head)."""
    sl, co = _i32(slots), _i32(cand_offsets)
    _check("onetrans_stage2_score", lib.onetrans_stage2_score(
        model.handle, cache.handle, sl, len(slots), co, _ptr(ns_tokens), _ptr(ns_out), _ptr(logits), _ptr(ws),
        ws.numel(), _stream(stream)))


def onetrans_cache_append(model: Model, cache: Cache, slots: Sequence[int], events: torch.Tensor,
                          types: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    sl = _i32(slots)
    _check("onetrans_cache_append", lib.onetrans_cache_append(
        model.handle, cache.handle, sl, len(slots), _ptr(events), _ptr(types), events.shape[1], _ptr(ws),
        ws.numel(), _stream(stream)))


def onetrans_forward(model: Model, x0: torch.Tensor, out: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    _check("onetrans_forward", lib.onetrans_forward(
        model.handle, _ptr(x0), x0.shape[0], x0.shape[1] - model.L_NS, _ptr(out), _ptr(ws), ws.numel(),
        _stream(stream)))


def model_from_arrays(shape, weights: Dict, pyramid_q=None, mode: int = BF16, device="cuda",
                      event_dim: int = 0) -> Model:
    """Copy a dict of NumPy weight arrays (the layout of onetrans.h) to the
    device and create a Model.  `shape` provides n_layers, d, n_heads, d_ff,
    L_NS, ns_feat, ns_hidden, n_types and eps."""
    import numpy as np
    dt = torch.bfloat16 if mode == BF16 else torch.float32

    def dev(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device=device, dtype=dt)

    tw = {}
    for k, v in weights.items():
        if k == "sep":
            continue
        tw[k] = [dev(a) for a in v] if isinstance(v, list) else dev(v)
    n_beh = len(weights.get("Wb1", [])) if event_dim else 0
    return Model(n_layers=shape.n_layers, d_model=shape.d, n_heads=shape.n_heads, d_ff=shape.d_ff,
                 L_NS=shape.L_NS, weights=tw, pyramid_q=pyramid_q, mode=mode,
                 ns_feat_dim=shape.ns_feat, ns_hidden=shape.ns_hidden, n_behaviors=n_beh,
                 event_dim=event_dim, rms_eps=shape.eps)


def onetrans_forward_backward(model: Model, x0: torch.Tensor, dy: torch.Tensor, out: torch.Tensor,
                              dx0: torch.Tensor, grads: Dict[str, Sequence[torch.Tensor]], ws: torch.Tensor,
                              stream=None) -> None:
    """x0 [B, L_S + L_NS, d] (model dtype); dy, out [B, L'_N, d] and dx0 [B, L_S + L_NS, d] float32;
    grads maps each block-stack weight name to per-layer float32 tensors of the weight's shape."""
    B, L0, _ = x0.shape
    g = Grads()
    keep = []
    for f in _WEIGHT_FIELDS:
        arr = (P * model.n_layers)(*[_ptr(t) for t in grads[f]])
        keep.append(arr)
        setattr(g, f, ctypes.cast(arr, PP))
    _check("onetrans_forward_backward", lib.onetrans_forward_backward(
        model.handle, _ptr(x0), B, L0 - model.L_NS, _ptr(dy), _ptr(out), _ptr(dx0), ctypes.byref(g), _ptr(ws),
        ws.numel(), _stream(stream)))
