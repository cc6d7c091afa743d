"""Shared test helpers: build a model on the device from seeded synthetic
weights, run the oracle on the same (already rounded) arrays, compare."""
from __future__ import annotations

import dataclasses

import numpy as np

from onetrans_synth import ModelShape, make_weights

EPS = 1e-6
TOL = {"bf16": 2e-2, "fp32": 1e-4}   # max-abs-error / RMS(reference)


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    rms = np.sqrt(np.mean(ref * ref))
    return float(np.max(np.abs(got - ref)) / rms)


# A value the bf16 path stores in bf16 (the K/V cache, tokenizer outputs)
# carries, besides the computation's error, its own rounding (half an ulp,
# 2^-9 of its magnitude) and that of the bf16 operand it was computed from:
# its bar adds STORE_ULP * |x| per element to TOL * RMS.  Float32 outputs
# (the stack's final rows) keep the plain bar.
STORE_ULP = {"bf16": 2.0 ** -8, "fp32": 0.0}


def stored_err(got, ref, dtype) -> float:
    """max_i |got_i - ref_i| / (RMS(ref) + |ref_i| * STORE_ULP / TOL): at most
    TOL[dtype] exactly when every element is within TOL * RMS + STORE_ULP * |ref_i|."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    rms = np.sqrt(np.mean(ref * ref))
    return float(np.max(np.abs(got - ref) / (rms + np.abs(ref) * STORE_ULP[dtype] / TOL[dtype])))


def shape(n_layers=2, d=256, H=4, dff=1024, L_NS=12, F=512, Hh=None, n_types=3):
    return ModelShape(n_layers=n_layers, d=d, n_heads=H, d_ff=dff, L_NS=L_NS, ns_feat=F,
                      ns_hidden=Hh if Hh is not None else L_NS * d,
                      behavior_dims=tuple([64] * n_types))


def to_dev(a, dtype, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device=device, dtype=dtype)


def to_np(t):
    import torch
    return t.detach().to(torch.float32).cpu().numpy()


@dataclasses.dataclass
class Built:
    shape: ModelShape
    W: dict
    model: object
    dtype: str


def attn_std(d: int) -> float:
    """Weight scale at which attention is far from uniform: with RMS-normed
    rows, q and k entries come out ~N(0, 1) and the scores q.k/sqrt(d_h)
    ~N(0, 1), so a kernel that got the scores or the mask wrong moves the
    output well past the tolerance (at std 0.02 the scores are ~0.01 and a
    softmax that ignores them stays inside it)."""
    return 1.0 / float(np.sqrt(d))


def build(sh, seed, dtype="bf16", pyramid=None, event_dim=0, std=0.02, tweak=None):
    """Seeded weights -> model on the device.  `tweak(W)` may edit the weight
    dict in place before the model is made (the oracle reads the same dict)."""
    import unified_transformer_recommender_b200 as ot
    W = make_weights(sh, seed, dtype, event_dim=event_dim, std=std)
    if tweak is not None:
        tweak(W)
    mode = ot.BF16 if dtype == "bf16" else ot.FP32
    model = ot.model_from_arrays(sh, W, pyramid_q=pyramid, mode=mode, event_dim=event_dim)
    return Built(sh, W, model, dtype)


def tdt(dtype):
    import torch
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def run_forward(b, X0):
    """onetrans_forward of X0 [B, L0, d] through the C ABI; float32 [B, L'_N, d]."""
    import torch
    import unified_transformer_recommender_b200 as ot
    m = b.model
    L_S = X0.shape[1] - b.shape.L_NS
    sched = m.schedule(L_S)
    out = torch.empty(X0.shape[0], sched[-1], b.shape.d, dtype=torch.float32, device="cuda")
    ws = m.workspace(ot.OP_FORWARD, X0.shape[0], L_S)
    ot.onetrans_forward(m, to_dev(X0, tdt(b.dtype)), out, ws)
    torch.cuda.synchronize()
    return to_np(out)


def run_stage12(b, S, NS_tok, offsets, slots=None):
    """Stage I of S [U, L_S, d] into a fresh cache, then Stage II of NS_tok
    [C, L_NS, d] with the CSR `offsets`; returns (cache, ns_out [C, L_NS, d])."""
    import torch
    import unified_transformer_recommender_b200 as ot
    m = b.model
    U, L_S, d = S.shape
    slots = list(range(U)) if slots is None else slots
    cache = ot.Cache(m, max(slots) + 1, L_S + 64)
    ws1 = m.workspace(ot.OP_STAGE1, U, L_S)
    ot.onetrans_stage1_encode(m, cache, slots, to_dev(S, tdt(b.dtype)), ws1)
    C = NS_tok.shape[0]
    out = torch.empty(C, b.shape.L_NS, d, dtype=torch.float32, device="cuda")
    ws2 = m.workspace(ot.OP_STAGE2, C, L_S)
    ot.onetrans_stage2_score(m, cache, slots, offsets, to_dev(NS_tok, tdt(b.dtype)), out, ws2)
    torch.cuda.synchronize()
    return cache, to_np(out)
