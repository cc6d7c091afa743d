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


def build(sh, seed, dtype="bf16", pyramid=None, event_dim=0, std=0.02):
    import unified_transformer_recommender_b200 as ot
    W = make_weights(sh, seed, dtype, event_dim=event_dim, std=std)
    mode = ot.BF16 if dtype == "bf16" else ot.FP32
    model = ot.model_from_arrays(sh, W, pyramid_q=pyramid, mode=mode, event_dim=event_dim)
    return Built(sh, W, model, dtype)
