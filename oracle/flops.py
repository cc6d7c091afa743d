"""Analytic FLOP counts of the OneTrans hot path (test infrastructure only).

Counts are multiply-add pairs x 2 over the work the method defines; masked
(causally hidden) score entries are excluded, softmax exponentials are not
counted.  Sources as in oracle.onetrans: [FR] = fun-rec mdbook 7.5 "OneTrans:
Unifying Sequence Modeling and Feature Interaction".
"""
from __future__ import annotations

from typing import Optional, Sequence

from .onetrans import s_schedule


def _attn(d: int, key_counts) -> int:
    # q.k and p.v: 2 * d each per visible key
    return 4 * d * sum(key_counts)


def forward_flops(L_S: int, L_NS: int, d: int, d_ff: int, n_layers: int,
                  schedule: Optional[Sequence[int]] = None) -> dict:
    """Per-sample FLOPs of the stack on [S; NS] ([FR] 7.5.2 complexity:
    attention O(L L' d), FFN O(L' d^2))."""
    L = L_S + L_NS
    proj = attn = 0
    for n in range(n_layers):
        Lq = L if schedule is None else int(schedule[n])
        proj += 2 * L * 2 * d * d + 2 * Lq * d * d      # K,V all rows; Q tail rows
        attn += _attn(d, [p + 1 for p in range(L - Lq, L)])
        proj += 2 * Lq * d * d + 2 * Lq * 2 * d * d_ff  # W^O and the FFN on tail rows
        L = Lq
    return {"proj": proj, "attn": attn, "total": proj + attn}


def stage1_flops(L_S: int, L_NS: int, d: int, d_ff: int, n_layers: int,
                 schedule: Optional[Sequence[int]] = None) -> dict:
    """Per-user FLOPs of Stage I (S rows only)."""
    proj = attn = 0
    for s, sq in s_schedule(L_S, L_NS, n_layers, schedule):
        proj += 2 * s * 2 * d * d + 2 * sq * d * d + 2 * sq * d * d + 2 * sq * 2 * d * d_ff
        attn += _attn(d, [p + 1 for p in range(s - sq, s)])
    return {"proj": proj, "attn": attn, "total": proj + attn}


def stage2_flops(L_S: int, L_NS: int, d: int, d_ff: int, n_layers: int,
                 F: int, H: int, schedule: Optional[Sequence[int]] = None) -> dict:
    """Per-candidate FLOPs of Stage II, auto-split tokenizer included."""
    tok = 2 * (F * H + H * L_NS * d)
    proj = attn = 0
    for s, _ in s_schedule(L_S, L_NS, n_layers, schedule):
        proj += L_NS * (2 * 3 * d * d + 2 * d * d + 2 * 2 * d * d_ff)
        attn += _attn(d, [s + j + 1 for j in range(L_NS)])
    return {"tokenize": tok, "proj": proj, "attn": attn, "total": tok + proj + attn}


def append_flops(L_S_old: int, dL: int, d: int, d_ff: int, n_layers: int,
                 event_dim: int) -> dict:
    """Per-user FLOPs of one cross-request append of dL events (non-pyramid)."""
    tok = 2 * dL * (event_dim * d + d * d)
    proj = dL * n_layers * (2 * 3 * d * d + 2 * d * d + 2 * 2 * d * d_ff)
    attn = n_layers * _attn(d, [L_S_old + t + 1 for t in range(dL)])
    return {"tokenize": tok, "proj": proj, "attn": attn, "total": tok + proj + attn}


# --------------------------------------------------------------------------
# The worked answers printed with the practice problems ([FR] 7.5, Chinese
# edition, answers to problems 7.5.3 and 7.5.4).
# --------------------------------------------------------------------------

def pyramid_attention_ratio(L: float, n_layers: int, shrink_keys: bool) -> float:
    """Pyramid attention work over a full-length stack of the same depth when
    each layer halves the query count.  With keys kept at L the sum is
    L (L/2 + L/4 + ...) against n_layers L^2; with keys shrinking with the
    layer input the ratio is lower."""
    full = n_layers * L * L
    pyr, keys, Lq = 0.0, float(L), float(L)
    for _ in range(n_layers):
        Lq = Lq / 2.0
        pyr += keys * Lq
        if shrink_keys:
            keys = Lq
    return pyr / full


def kv_cache_ratio(C: int, L_S: int, L_NS: int) -> float:
    """Sequence work without and with the cross-candidate cache:
    O(C L_S) against O(L_S + C L_NS)."""
    return (C * L_S) / (L_S + C * L_NS)
