"""fp64 CPU oracle of the OneTrans block stack and its two-stage KV-cached scoring.

TEST INFRASTRUCTURE ONLY.  This module is the independent reference that the
CUDA path is checked against.  Only the test-suite, the smoke check and the
benchmark's CPU-baseline leg may import it; the product path never does.  It
shares no code with the CUDA library: it is plain NumPy in float64, written
from the method's description, with no blocking, fusion or reordering.

Sources (cited by page title and section):
  [FR]  fun-rec mdbook 7.5, "OneTrans: Unifying Sequence Modeling and Feature
        Interaction" (English edition; the Chinese edition carries the same
        equations and the worked answers of the practice problems).
  [PD]  paper-daily deep reading, "OneTrans: Unified Feature Interaction and
        Sequence Modeling with One Transformer in Industrial Recommender".
  [LP]  listeners-pseudolab review notes, "OneTrans 정리".

Readings where the pages are silent (each also listed in the design notes):
  * W^O: one shared d x d output projection for every token, no bias.
  * QKV have no bias ([FR] 7.5.1 eq. for (q_i, k_i, v_i)); the FFN has b1, b2.
  * RMSNorm: x * (mean(x^2) + eps)^(-1/2) * g, one gain per sublayer per
    layer shared by S and NS rows; no final norm, no positional encoding.
  * Heads are contiguous d_h slices; scale 1/sqrt(d_h); no dropout.
  * Causal predicate: key index <= query index, positions relative to the
    layer's input rows (NS rows come after S rows).
  * Stage II: one softmax over the union [cached S keys; own NS keys 0..j].
  * Append is defined for non-pyramid stacks only.

Every function works on float64 copies of its inputs.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence

import numpy as np

F64 = np.float64


def _f(x) -> np.ndarray:
    return np.asarray(x, dtype=F64)


# --------------------------------------------------------------------------
# Elementwise pieces
# --------------------------------------------------------------------------

def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """Pre-norm RMSNorm of each row ([FR] 7.5.1, "Pre-norm + RMSNorm")."""
    x = _f(x)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * _f(g)


def gelu_tanh(x: np.ndarray) -> np.ndarray:
    """phi of the mixed FFN: the tanh form of GELU (Hendrycks & Gimpel, 2016)."""
    x = _f(x)
    return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)))


# --------------------------------------------------------------------------
# Attention over a query subset with the causal predicate
# --------------------------------------------------------------------------

def masked_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                     q_pos: np.ndarray, n_heads: int) -> np.ndarray:
    """Multi-head softmax attention of queries q[i] at key positions q_pos[i].

    q: [Lq, d]; k, v: [Lk, d]; q_pos: [Lq] ints.  Query i sees keys
    0..q_pos[i] ([FR] 7.5.1 "Mixed Causal Attention": S rows see earlier S rows,
    NS rows see every S row and earlier NS rows).  Heads are contiguous d_h
    slices, concatenated back into d.
    """
    q, k, v = _f(q), _f(k), _f(v)
    Lq, d = q.shape
    Lk = k.shape[0]
    dh = d // n_heads
    out = np.empty((Lq, d), dtype=F64)
    visible = np.arange(Lk)[None, :] <= np.asarray(q_pos)[:, None]
    for h in range(n_heads):
        sl = slice(h * dh, (h + 1) * dh)
        s = q[:, sl] @ k[:, sl].T / np.sqrt(dh)
        s = np.where(visible, s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, sl] = p @ v[:, sl]
    return out


# --------------------------------------------------------------------------
# One OneTrans block on one sample
# --------------------------------------------------------------------------

def _row_weights(W: Dict, l: int, n_S: int, i: int):
    """Mixed parameterization: row i < n_S uses the shared S set, row n_S + j
    uses the set of NS token j ([FR] 7.5.1, conditional W_i^Psi)."""
    if i < n_S:
        return (W["Wqkv_S"][l], W["W1_S"][l], W["b1_S"][l], W["W2_S"][l], W["b2_S"][l])
    j = i - n_S
    return (W["Wqkv_NS"][l][j], W["W1_NS"][l][j], W["b1_NS"][l][j],
            W["W2_NS"][l][j], W["b2_NS"][l][j])


def qkv_rows(h: np.ndarray, W: Dict, l: int, n_S: int, rows: Sequence[int]):
    """(q_i, k_i, v_i) = (W_i^Q h_i, W_i^K h_i, W_i^V h_i) for the given rows.

    Rows sharing a weight set (all S rows) are done as one matrix product;
    each NS row uses its own set."""
    d = h.shape[1]
    rows = list(rows)
    y = np.empty((len(rows), 3 * d))
    s_idx = [t for t, i in enumerate(rows) if i < n_S]
    if s_idx:
        y[s_idx] = h[[rows[t] for t in s_idx]] @ _f(W["Wqkv_S"][l]).T
    for t, i in enumerate(rows):
        if i >= n_S:
            y[t] = _f(W["Wqkv_NS"][l][i - n_S]) @ h[i]
    return y[:, :d], y[:, d:2 * d], y[:, 2 * d:]


def mixed_ffn_rows(h: np.ndarray, W: Dict, l: int, n_S: int,
                   row_ids: Sequence[int]) -> np.ndarray:
    """MixedFFN(h_i) = W_i^2 phi(W_i^1 h_i + b_i^1) + b_i^2 ([FR] 7.5.1 "Mixed FFN").

    h holds one row per entry of row_ids, the row's position in the layer
    input, which selects the weight set.  S rows share one set and are done as
    one matrix product; each NS row uses its own set."""
    row_ids = list(row_ids)
    out = np.empty_like(h)
    s_idx = [t for t, i in enumerate(row_ids) if i < n_S]
    if s_idx:
        out[s_idx] = mlp2(h[s_idx], W["W1_S"][l], W["b1_S"][l], W["W2_S"][l], W["b2_S"][l])
    for t, i in enumerate(row_ids):
        if i >= n_S:
            _, W1, b1, W2, b2 = _row_weights(W, l, n_S, i)
            out[t] = mlp2(h[t], W1, b1, W2, b2)
    return out


def block(x: np.ndarray, W: Dict, l: int, L_NS: int, Lq: int, n_heads: int,
          eps: float) -> np.ndarray:
    """One pre-norm OneTrans block on one sample, keeping the tail Lq rows.

    x: [L, d], the layer input (S rows then the L_NS NS rows).  Keys/values
    come from all L rows, queries only from the tail index set
    Q = {L - Lq + 1, ..., L} (1-based; [FR] 7.5.2), and the output holds the
    Lq tail rows:
        h      = RMSNorm(x; g_attn)
        a_Q    = Attn(q_Q, k_all, v_all) with the causal predicate
        x'_Q   = x_Q + W^O a_Q
        out_Q  = x'_Q + MixedFFN(RMSNorm(x'_Q; g_ffn))
    """
    x = _f(x)
    L, d = x.shape
    n_S = L - L_NS
    tail = list(range(L - Lq, L))
    h = rmsnorm(x, W["g_attn"][l], eps)
    _, k, v = qkv_rows(h, W, l, n_S, range(L))
    q, _, _ = qkv_rows(h, W, l, n_S, tail)
    a = masked_attention(q, k, v, np.asarray(tail), n_heads)
    x1 = x[tail] + a @ _f(W["Wo"][l]).T
    h2 = rmsnorm(x1, W["g_ffn"][l], eps)
    return x1 + mixed_ffn_rows(h2, W, l, n_S, tail)


def forward(X0: np.ndarray, W: Dict, L_NS: int, n_heads: int, eps: float,
            schedule: Optional[Sequence[int]] = None) -> np.ndarray:
    """The OneTrans stack on X^(0) = [S-tokens; NS-tokens] ([FR] 7.5.0 eq. for
    X^(0), 7.5.2 pyramid).  X0: [B, L0, d]; schedule[n] = L'_n (None keeps every
    row).  Returns [B, L'_N, d]."""
    X0 = _f(X0)
    N = len(W["Wo"])
    outs = []
    for b in range(X0.shape[0]):
        x = X0[b]
        for l in range(N):
            Lq = x.shape[0] if schedule is None else int(schedule[l])
            x = block(x, W, l, L_NS, Lq, n_heads, eps)
        outs.append(x)
    return np.stack(outs)


# --------------------------------------------------------------------------
# Tokenizers
# --------------------------------------------------------------------------

def mlp2(x: np.ndarray, W1, b1, W2, b2) -> np.ndarray:
    """Two-layer MLP, Linear -> GELU-tanh -> Linear, on the last axis."""
    return gelu_tanh(_f(x) @ _f(W1).T + _f(b1)) @ _f(W2).T + _f(b2)


def autosplit(feats: np.ndarray, W: Dict, L_NS: int) -> np.ndarray:
    """Auto-Split tokenizer ([FR] 7.5.0 eq. for NS-tokens):
    NS-tokens = Split(MLP(Concat(NS)), L_NS).  feats: [N, F] (already
    concatenated).  Returns [N, L_NS, d]; token t is MLP output columns
    [t d, (t+1) d)."""
    y = mlp2(feats, W["Wa1"], W["ba1"], W["Wa2"], W["ba2"])
    n = y.shape[0]
    return y.reshape(n, L_NS, y.shape[1] // L_NS)


def tokenize_groupwise(groups: Sequence[np.ndarray], G: Dict) -> np.ndarray:
    """Group-wise NS tokenizer ([PD] 2.1 "Unified Tokenization"; [LP] 3.1
    "Non-Sequential Token (NS)"): the non-sequential features come split into
    semantic groups (user profile, item attributes, ...); group g, its
    features concatenated, goes through its own two-layer MLP and becomes NS
    token g.  groups[g]: [N, F_g]; G: Wg1/bg1/Wg2/bg2 lists indexed by group.
    Returns [N, L_NS, d] with L_NS = the number of groups."""
    toks = [mlp2(x, G["Wg1"][g], G["bg1"][g], G["Wg2"][g], G["bg2"][g])
            for g, x in enumerate(groups)]
    return np.stack(toks, axis=1)


def tokenize_events(events: np.ndarray, types: np.ndarray, W: Dict) -> np.ndarray:
    """Per-behavior MLP alignment plus an additive behavior-type identifier
    ([FR] 7.5.0, MLP_i(e_ij) and the timestamp-aware merge's type ids).
    events: [..., e]; types: [...] ints.  Returns [..., d]."""
    ev = _f(events)
    ty = np.asarray(types)
    flat_e = ev.reshape(-1, ev.shape[-1])
    flat_t = ty.reshape(-1)
    d = _f(W["type_emb"]).shape[1]
    out = np.empty((flat_e.shape[0], d))
    for r in range(flat_e.shape[0]):
        t = int(flat_t[r])
        out[r] = mlp2(flat_e[r], W["Wb1"][t], W["bb1"][t], W["Wb2"][t], W["bb2"][t]) \
            + _f(W["type_emb"][t])
    return out.reshape(ty.shape + (d,))


def merge_intent_order(seqs: List[np.ndarray], W: Dict) -> np.ndarray:
    """Timestamp-agnostic merge ([FR] 7.5.0): behavior-specific MLPs align each
    sequence to d, sequences are laid out in the given intent order with one
    learnable [SEP] between consecutive sequences.  seqs[i]: [L_i, e_i].
    Returns [L_S, d] with L_S = sum_i L_i + (n - 1)."""
    parts = []
    for i, s in enumerate(seqs):
        if i:
            parts.append(_f(W["sep"])[None, :])
        parts.append(mlp2(s, W["Wb1"][i], W["bb1"][i], W["Wb2"][i], W["bb2"][i]))
    return np.concatenate(parts, axis=0)


def score_head(h_ns: np.ndarray, W: Dict) -> np.ndarray:
    """Optional scoring head on the final NS states.  The pages hand the final
    NS rows downstream as the compact representation of the candidate
    ([FR] 7.5.2) and give no head; the reading here is one linear unit over
    their concatenation: logit = w_head . vec(h_NS) + b_head, vec() taking
    token 0's d entries first.  h_ns: [..., L_NS, d].  Returns [...]."""
    h = _f(h_ns)
    flat = h.reshape(h.shape[:-2] + (h.shape[-2] * h.shape[-1],))
    return flat @ _f(W["w_head"]) + _f(W["b_head"])[0]


# --------------------------------------------------------------------------
# Two-stage KV-cached serving
# --------------------------------------------------------------------------

def s_schedule(L_S: int, L_NS: int, n_layers: int,
               schedule: Optional[Sequence[int]]) -> List[tuple]:
    """(s_n, s'_n) per layer: S rows in the layer input and S rows among its
    tail queries, s'_n = max(L'_n - L_NS, 0)."""
    out, s = [], L_S
    for l in range(n_layers):
        Lq = s + L_NS if schedule is None else int(schedule[l])
        sq = max(Lq - L_NS, 0)
        out.append((s, sq))
        s = sq
    return out


def stage1(S: np.ndarray, W: Dict, L_NS: int, n_heads: int, eps: float,
           schedule: Optional[Sequence[int]] = None) -> List[tuple]:
    """Stage I ([FR] 7.5.3): run the S rows of one user through the stack and
    keep each layer's S-side keys and values.  Causality makes the S rows
    independent of the NS rows, so the NS rows are never formed.
    S: [L_S, d].  Returns [(K_n, V_n)] with K_n, V_n: [s_n, d]."""
    x = _f(S)
    N = len(W["Wo"])
    cache = []
    for l, (s, sq) in enumerate(s_schedule(x.shape[0], L_NS, N, schedule)):
        h = rmsnorm(x, W["g_attn"][l], eps)
        _, k, v = qkv_rows(h, W, l, s, range(s))
        cache.append((k, v))
        if sq == 0:
            x = x[:0]
            continue
        tail = list(range(s - sq, s))
        q, _, _ = qkv_rows(h, W, l, s, tail)
        a = masked_attention(q, k, v, np.asarray(tail), n_heads)
        x1 = x[tail] + a @ _f(W["Wo"][l]).T
        x = x1 + mixed_ffn_rows(rmsnorm(x1, W["g_ffn"][l], eps), W, l, s, tail)
    return cache


def stage2(cache: List[tuple], NS: np.ndarray, W: Dict, n_heads: int,
           eps: float) -> np.ndarray:
    """Stage II ([FR] 7.5.3): the NS rows of one candidate against the cached
    S-side keys/values.  Per layer, NS token j attends, in one softmax, to the
    s_n cached S keys and its own NS keys 0..j, then goes through its own FFN.
    NS: [L_NS, d].  Returns the final NS rows [L_NS, d]."""
    x = _f(NS)
    L_NS = x.shape[0]
    for l, (Ks, Vs) in enumerate(cache):
        s = Ks.shape[0]
        h = rmsnorm(x, W["g_attn"][l], eps)
        rows = list(range(L_NS))
        q = np.empty_like(h); k = np.empty_like(h); v = np.empty_like(h)
        for j in rows:
            y = _f(W["Wqkv_NS"][l][j]) @ h[j]
            d = h.shape[1]
            q[j], k[j], v[j] = y[:d], y[d:2 * d], y[2 * d:]
        K = np.concatenate([Ks, k]); V = np.concatenate([Vs, v])
        a = masked_attention(q, K, V, np.arange(s, s + L_NS), n_heads)
        x1 = x + a @ _f(W["Wo"][l]).T
        h2 = rmsnorm(x1, W["g_ffn"][l], eps)
        x = x1 + mixed_ffn_rows(h2, W, l, s, [s + j for j in rows])
    return x


def append(cache: List[tuple], new_S: np.ndarray, W: Dict, n_heads: int,
           eps: float) -> List[tuple]:
    """Cross-request cache append ([FR] 7.5.3): only the dL new S rows are run
    through the (non-pyramid) stack; at each layer their keys/values are
    concatenated after the cached ones and their queries attend causally to
    old and new keys.  new_S: [dL, d].  Returns the extended cache."""
    x = _f(new_S)
    dL = x.shape[0]
    out = []
    for l, (Ks, Vs) in enumerate(cache):
        s_old = Ks.shape[0]
        s = s_old + dL
        h = rmsnorm(x, W["g_attn"][l], eps)
        d = h.shape[1]
        y = h @ _f(W["Wqkv_S"][l]).T
        q, k, v = y[:, :d], y[:, d:2 * d], y[:, 2 * d:]
        K = np.concatenate([Ks, k]); V = np.concatenate([Vs, v])
        out.append((K, V))
        a = masked_attention(q, K, V, np.arange(s_old, s), n_heads)
        x1 = x + a @ _f(W["Wo"][l]).T
        x = x1 + mixed_ffn_rows(rmsnorm(x1, W["g_ffn"][l], eps), W, l, s,
                                range(s_old, s))
    return out


# --------------------------------------------------------------------------
# Backward pass (training: gradients of the block stack)
# --------------------------------------------------------------------------
#
# The pages train the stack end to end and speed it up by recomputing
# activations in the backward pass ([FR] 7.5.3 system optimizations; [PD]
# 4.3, the "+ mixed precision + recomputation" row).  The oracle gives the
# exact gradient by the chain rule, step by step in reverse order of
# `block`; it keeps each layer's input and recomputes the layer's
# intermediates, the recomputation scheme itself.  The upstream gradient dY
# of the stack's output defines the loss: L = sum(dY * Y).

_GRAD_KEYS = ("g_attn", "g_ffn", "Wqkv_S", "Wqkv_NS", "Wo", "W1_S", "b1_S", "W2_S",
              "b2_S", "W1_NS", "b1_NS", "W2_NS", "b2_NS")


def rmsnorm_backward(x: np.ndarray, g: np.ndarray, eps: float, dy: np.ndarray):
    """Gradients of y = x r g, r = (mean(x^2) + eps)^(-1/2), over rows x.
    Returns (dx, dg): dx = r (g dy) - x r^3 sum(g dy x) / d, dg = sum_rows dy x r."""
    x, g, dy = _f(x), _f(g), _f(dy)
    d = x.shape[-1]
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    gy = dy * g
    dx = r * gy - x * r ** 3 * np.sum(gy * x, axis=-1, keepdims=True) / d
    dg = np.sum(dy * x * r, axis=tuple(range(x.ndim - 1)))
    return dx, dg


def gelu_tanh_grad(x: np.ndarray) -> np.ndarray:
    """d/dx of 0.5 x (1 + tanh(c (x + 0.044715 x^3))), c = sqrt(2/pi)."""
    x = _f(x)
    c = np.sqrt(2.0 / np.pi)
    t = np.tanh(c * (x + 0.044715 * x ** 3))
    return 0.5 * (1.0 + t) + 0.5 * x * (1.0 - t * t) * c * (1.0 + 3 * 0.044715 * x * x)


def masked_attention_backward(q, k, v, q_pos, n_heads: int, do: np.ndarray):
    """Gradients of masked_attention with respect to q, k, v for the output
    gradient do [Lq, d].  Per head, with P the softmax of the masked scores:
    dV = P^T dO, dP = dO V^T, dS = P (dP - rowsum(dP P)), dQ = dS K / sqrt(d_h),
    dK = dS^T Q / sqrt(d_h)."""
    q, k, v, do = _f(q), _f(k), _f(v), _f(do)
    Lq, d = q.shape
    Lk = k.shape[0]
    dh = d // n_heads
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    visible = np.arange(Lk)[None, :] <= np.asarray(q_pos)[:, None]
    for h in range(n_heads):
        sl = slice(h * dh, (h + 1) * dh)
        s = np.where(visible, q[:, sl] @ k[:, sl].T / np.sqrt(dh), -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        dv[:, sl] = p.T @ do[:, sl]
        dp = do[:, sl] @ v[:, sl].T
        ds = p * (dp - np.sum(dp * p, axis=1, keepdims=True))
        dq[:, sl] = ds @ k[:, sl] / np.sqrt(dh)
        dk[:, sl] = ds.T @ q[:, sl] / np.sqrt(dh)
    return dq, dk, dv


def _zero_grads(W: Dict, l: int) -> Dict:
    return {key: np.zeros(np.shape(W[key][l])) for key in _GRAD_KEYS}


def block_backward(x: np.ndarray, W: Dict, l: int, L_NS: int, Lq: int, n_heads: int,
                   eps: float, dy: np.ndarray):
    """Gradient of `block` (one sample, layer l) for the output gradient
    dy [Lq, d].  Recomputes the block's intermediates from its input x [L, d]
    and returns (dx [L, d], grads of layer l's weights keyed like W)."""
    x, dy = _f(x), _f(dy)
    L, d = x.shape
    n_S = L - L_NS
    tail = list(range(L - Lq, L))
    G = _zero_grads(W, l)
    # ---- recompute the forward
    h = rmsnorm(x, W["g_attn"][l], eps)
    _, k, v = qkv_rows(h, W, l, n_S, range(L))
    q, _, _ = qkv_rows(h, W, l, n_S, tail)
    a = masked_attention(q, k, v, np.asarray(tail), n_heads)
    x1 = x[tail] + a @ _f(W["Wo"][l]).T
    h2 = rmsnorm(x1, W["g_ffn"][l], eps)
    # ---- y = x1 + MixedFFN(h2): per row, the row's weight set
    dx1 = dy.copy()
    dh2 = np.empty_like(h2)
    for t, i in enumerate(tail):
        _, W1, b1, W2, _ = _row_weights(W, l, n_S, i)
        u = _f(W1) @ h2[t] + _f(b1)
        z = gelu_tanh(u)
        du = (_f(W2).T @ dy[t]) * gelu_tanh_grad(u)
        dh2[t] = _f(W1).T @ du
        if i < n_S:
            G["W2_S"] += np.outer(dy[t], z); G["b2_S"] += dy[t]
            G["W1_S"] += np.outer(du, h2[t]); G["b1_S"] += du
        else:
            j = i - n_S
            G["W2_NS"][j] += np.outer(dy[t], z); G["b2_NS"][j] += dy[t]
            G["W1_NS"][j] += np.outer(du, h2[t]); G["b1_NS"][j] += du
    dxn, G["g_ffn"] = rmsnorm_backward(x1, W["g_ffn"][l], eps, dh2)
    dx1 += dxn
    # ---- x1 = x[tail] + W^O a
    G["Wo"] = dx1.T @ a
    da = dx1 @ _f(W["Wo"][l])
    dx = np.zeros_like(x)
    dx[tail] += dx1
    # ---- attention, then (q, k, v) = W_i^{Q,K,V} h_i per row
    dq, dk, dv = masked_attention_backward(q, k, v, np.asarray(tail), n_heads, da)
    dqkv = np.zeros((L, 3 * d))
    dqkv[tail, :d] = dq
    dqkv[:, d:2 * d] = dk
    dqkv[:, 2 * d:] = dv
    dh = np.empty_like(h)
    for i in range(L):
        Wi = _f(W["Wqkv_S"][l] if i < n_S else W["Wqkv_NS"][l][i - n_S])
        dh[i] = Wi.T @ dqkv[i]
        if i < n_S:
            G["Wqkv_S"] += np.outer(dqkv[i], h[i])
        else:
            G["Wqkv_NS"][i - n_S] += np.outer(dqkv[i], h[i])
    dxh, G["g_attn"] = rmsnorm_backward(x, W["g_attn"][l], eps, dh)
    dx += dxh
    return dx, G


def forward_backward(X0: np.ndarray, W: Dict, L_NS: int, n_heads: int, eps: float,
                     schedule: Optional[Sequence[int]], dY: np.ndarray):
    """Forward of the stack keeping only each layer's input, then the
    backward layer by layer, recomputing each layer from its input.
    X0 [B, L0, d], dY [B, L'_N, d].  Returns (Y, dX0, dW) with dW[key] a list
    over layers, summed over the batch."""
    X0, dY = _f(X0), _f(dY)
    N = len(W["Wo"])
    dW = {key: [np.zeros(np.shape(W[key][l])) for l in range(N)] for key in _GRAD_KEYS}
    Y, dX = [], []
    for b in range(X0.shape[0]):
        xs = [X0[b]]
        for l in range(N):
            Lq = xs[-1].shape[0] if schedule is None else int(schedule[l])
            xs.append(block(xs[-1], W, l, L_NS, Lq, n_heads, eps))
        Y.append(xs[-1])
        g = dY[b]
        for l in reversed(range(N)):
            Lq = xs[l + 1].shape[0]
            g, G = block_backward(xs[l], W, l, L_NS, Lq, n_heads, eps, g)
            for key in _GRAD_KEYS:
                dW[key][l] += G[key]
        dX.append(g)
    return np.stack(Y), np.stack(dX), dW
