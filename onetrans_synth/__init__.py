"""Seeded synthetic inputs and weights for the OneTrans block stack.

This module is shared by the CPU oracle and by the CUDA path's tests and
benchmark.  It holds none of the method's arithmetic: it only draws random
numbers (NumPy PCG64), rounds them to the storage precision, and states the
workload shapes.  Every tensor is returned as a float32 NumPy array; in bf16
mode the values are already rounded to bf16 (round-to-nearest-even), so the
oracle and the GPU consume bit-identical operands.

Shapes follow the OneTrans description (fun-rec mdbook 7.5, "OneTrans: Unifying
Sequence Modeling and Feature Interaction", sections 7.5.0-7.5.3): a merged
sequence of S-tokens followed by L_NS NS-tokens, d-wide, with one shared
weight set for S rows and one per NS token.

Weight layout (row-major, W[out][in], per layer l):
  g_attn[l], g_ffn[l]     [d]            RMSNorm gains, 1 + N(0, 0.02)
  Wqkv_S[l]               [3d, d]        rows: Q, then K, then V
  Wqkv_NS[l]              [L_NS, 3d, d]
  Wo[l]                   [d, d]         shared output projection, no bias
  W1_S[l], b1_S[l]        [dff, d], [dff]
  W2_S[l], b2_S[l]        [d, dff], [d]
  W1_NS[l], b1_NS[l]      [L_NS, dff, d], [L_NS, dff]
  W2_NS[l], b2_NS[l]      [L_NS, d, dff], [L_NS, d]
Tokenizer weights:
  Wa1 [H, F], ba1 [H], Wa2 [L_NS*d, H], ba2 [L_NS*d]   auto-split MLP
  Wb1[t] [d, e_t], bb1[t] [d], Wb2[t] [d, d], bb2[t] [d] per-behavior MLP
  type_emb [n_types, d], sep [d]
  w_head [L_NS*d], b_head [1]                          optional scoring head
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence

import numpy as np

__all__ = [
    "ModelShape", "Workload", "WORKLOADS", "bf16_round", "linear_pyramid",
    "make_weights", "gen_normal",
]


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); return float32."""
    a = np.ascontiguousarray(x, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    out = r.astype(np.uint32).view(np.float32)
    # keep NaN payloads quiet (inputs here are finite; this is a guard only)
    out = np.where(np.isnan(a), a, out)
    return out.reshape(a.shape)


def linear_pyramid(L0: int, L_min: int, n_layers: int) -> List[int]:
    """Query counts L'_n for n = 1..N falling linearly from L0 to L_min.

    Both endpoints are kept (layer 1 keeps every row, the last layer keeps
    L_min rows); interior values are rounded half-up in integer arithmetic:
        L'_n = L0 - floor((2 (L0 - L_min)(n - 1) + (N - 1)) / (2 (N - 1)))
    This is a workload shape, not part of the block's arithmetic.
    """
    if n_layers == 1:
        return [L_min]
    N = n_layers
    return [L0 - (2 * (L0 - L_min) * (n - 1) + (N - 1)) // (2 * (N - 1))
            for n in range(1, N + 1)]


@dataclasses.dataclass(frozen=True)
class ModelShape:
    n_layers: int
    d: int
    n_heads: int
    d_ff: int
    L_NS: int
    ns_feat: int          # F, width of the concatenated NS feature vector
    ns_hidden: int        # H, hidden width of the auto-split MLP
    behavior_dims: tuple  # raw event width per behavior type
    eps: float = 1e-6

    @property
    def d_h(self) -> int:
        return self.d // self.n_heads

    @property
    def n_types(self) -> int:
        return len(self.behavior_dims)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    shape: ModelShape
    L_S: int
    users: int
    cands: int                      # candidates per user (Stage II)
    pyramid: Optional[tuple]        # L'_n per layer, or None (all rows kept)
    dtype: str                      # "bf16" or "fp32"
    dL: int = 0                     # appended events per user
    event_dim: int = 0
    seed_inputs: int = 0
    seed_weights: int = 1000

    @property
    def L0(self) -> int:
        return self.L_S + self.shape.L_NS


_S6 = ModelShape(n_layers=6, d=256, n_heads=4, d_ff=1024, L_NS=12, ns_feat=512,
                 ns_hidden=3072, behavior_dims=(64, 64, 64))
_L8 = ModelShape(n_layers=8, d=384, n_heads=4, d_ff=1536, L_NS=16, ns_feat=512,
                 ns_hidden=16 * 384, behavior_dims=(64, 64, 64))
_TINY = ModelShape(n_layers=1, d=32, n_heads=2, d_ff=128, L_NS=4, ns_feat=40,
                   ns_hidden=4 * 32, behavior_dims=(16, 24))

WORKLOADS: Dict[str, Workload] = {
    # 1 layer, d=32; two behavior sequences (12 x 16, 11 x 24) merged in
    # intent order with one [SEP]: L_S = 12 + 11 + 1 = 24.
    "tiny": Workload("tiny", _TINY, L_S=24, users=2, cands=3, pyramid=None,
                     dtype="fp32", seed_inputs=0, seed_weights=0),
    # 6 x 256 pyramid forward over [S; NS] = 1178 + 12 rows, 64 users.
    "s_forward": Workload("s_forward", _S6, L_S=1178, users=64, cands=1,
                          pyramid=tuple(linear_pyramid(1190, 12, 6)),
                          dtype="bf16", seed_inputs=1, seed_weights=1001),
    # Stage I of 16 users x 1178 S rows; Stage II of 512 candidates per user.
    "kv_serving": Workload("kv_serving", _S6, L_S=1178, users=16, cands=512,
                           pyramid=tuple(linear_pyramid(1190, 12, 6)),
                           dtype="bf16", seed_inputs=2, seed_weights=1002),
    # Non-pyramid 6 x 256; 256 cached users, append 16 events, 128 candidates.
    "append": Workload("append", _S6, L_S=1178, users=256, cands=128,
                       pyramid=None, dtype="bf16", dL=16, event_dim=64,
                       seed_inputs=3, seed_weights=1003),
    # 8 x 384 pyramid forward over 2048 + 16 rows, 256 users.
    "l_forward": Workload("l_forward", _L8, L_S=2048, users=256, cands=1,
                          pyramid=tuple(linear_pyramid(2064, 16, 8)),
                          dtype="bf16", seed_inputs=4, seed_weights=1004),
}


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def _finish(a: np.ndarray, dtype: str) -> np.ndarray:
    a = a.astype(np.float32)
    return bf16_round(a) if dtype == "bf16" else a


def gen_normal(seed: int, shape, dtype: str, std: float = 1.0,
               mean: float = 0.0) -> np.ndarray:
    """N(mean, std^2) samples of the given shape, rounded to `dtype` storage."""
    r = _rng(seed)
    return _finish(mean + std * r.standard_normal(size=shape, dtype=np.float64), dtype)


def make_weights(shape: ModelShape, seed: int, dtype: str, event_dim: int = 0,
                 std: float = 0.02) -> Dict[str, object]:
    """All block-stack and tokenizer weights for `shape`, drawn in a fixed order.

    Matrices ~ N(0, std^2); biases ~ N(0, std^2); gains ~ 1 + N(0, std^2).
    Per-layer entries are lists indexed by layer.
    """
    r = _rng(seed)
    d, dff, L_NS, N = shape.d, shape.d_ff, shape.L_NS, shape.n_layers

    def nrm(*s):
        return _finish(std * r.standard_normal(size=s, dtype=np.float64), dtype)

    def gain(*s):
        return _finish(1.0 + std * r.standard_normal(size=s, dtype=np.float64), dtype)

    W: Dict[str, object] = {k: [] for k in (
        "g_attn", "g_ffn", "Wqkv_S", "Wqkv_NS", "Wo", "W1_S", "b1_S", "W2_S",
        "b2_S", "W1_NS", "b1_NS", "W2_NS", "b2_NS")}
    for _ in range(N):
        W["g_attn"].append(gain(d))
        W["g_ffn"].append(gain(d))
        W["Wqkv_S"].append(nrm(3 * d, d))
        W["Wqkv_NS"].append(nrm(L_NS, 3 * d, d))
        W["Wo"].append(nrm(d, d))
        W["W1_S"].append(nrm(dff, d))
        W["b1_S"].append(nrm(dff))
        W["W2_S"].append(nrm(d, dff))
        W["b2_S"].append(nrm(d))
        W["W1_NS"].append(nrm(L_NS, dff, d))
        W["b1_NS"].append(nrm(L_NS, dff))
        W["W2_NS"].append(nrm(L_NS, d, dff))
        W["b2_NS"].append(nrm(L_NS, d))
    H, F = shape.ns_hidden, shape.ns_feat
    W["Wa1"] = nrm(H, F)
    W["ba1"] = nrm(H)
    W["Wa2"] = nrm(L_NS * d, H)
    W["ba2"] = nrm(L_NS * d)
    dims = list(shape.behavior_dims)
    if event_dim:
        dims = [event_dim] * len(dims)
    W["Wb1"] = [nrm(d, e) for e in dims]
    W["bb1"] = [nrm(d) for _ in dims]
    W["Wb2"] = [nrm(d, d) for _ in dims]
    W["bb2"] = [nrm(d) for _ in dims]
    W["type_emb"] = nrm(len(dims), d)
    W["sep"] = nrm(d)
    # drawn last, so every weight above keeps the values of earlier versions
    W["w_head"] = nrm(L_NS * d)
    W["b_head"] = nrm(1)
    return W


def make_group_weights(d: int, group_dims: Sequence[int], group_hidden: Sequence[int], seed: int,
                       dtype: str, std: float = 0.02) -> Dict[str, List[np.ndarray]]:
    """Weights of a group-wise NS tokenizer, one two-layer MLP per feature group:
    Wg1[g] [h_g, F_g], bg1[g] [h_g], Wg2[g] [d, h_g], bg2[g] [d], drawn group
    by group from their own seed (the block-stack weights are untouched)."""
    r = _rng(seed)

    def nrm(*s):
        return _finish(std * r.standard_normal(size=s, dtype=np.float64), dtype)

    W: Dict[str, List[np.ndarray]] = {"Wg1": [], "bg1": [], "Wg2": [], "bg2": []}
    for F_g, h_g in zip(group_dims, group_hidden):
        W["Wg1"].append(nrm(h_g, F_g))
        W["bg1"].append(nrm(h_g))
        W["Wg2"].append(nrm(d, h_g))
        W["bg2"].append(nrm(d))
    return W


def tiny_raw_inputs(seed: int = 0) -> Dict[str, np.ndarray]:
    """Raw inputs of the tiny workload: two behavior sequences, NS features."""
    wl = WORKLOADS["tiny"]
    r = _rng(seed)
    U, C = wl.users, wl.cands
    seqs = [r.standard_normal(size=(U, 12, 16)).astype(np.float32),
            r.standard_normal(size=(U, 11, 24)).astype(np.float32)]
    feats = r.standard_normal(size=(U * C, wl.shape.ns_feat)).astype(np.float32)
    return {"seq0": seqs[0], "seq1": seqs[1], "feats": feats}


def random_types(seed: int, shape, n_types: int) -> np.ndarray:
    """Behavior type ids, uniform over {0..n_types-1}, int32."""
    return _rng(seed).integers(0, n_types, size=shape, dtype=np.int32)
