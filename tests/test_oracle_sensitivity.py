"""The GPU parity tests' weight scale can see attention mistakes.

Mistakes are planted in the oracle, on the CPU: a softmax that ignores the
scores (uniform over the visible keys), a causal mask that lets every query
see one key past its own position, and a Stage II whose NS tokens see all
of their candidate's own NS keys ([FR] 7.5.1 "Mixed Causal Attention", 7.5.3
Stage II).  At weight std 1/sqrt(d), the scale of `test_gpu_attention.py`,
each moves the output by more than twice the bf16 tolerance of the parity
tests, so a kernel with that mistake fails them.  At std 0.02 the scores are
~0.01 and the same mistakes stay inside the tolerance."""
import numpy as np
import pytest

from onetrans_synth import gen_normal, make_weights
from oracle import onetrans as O
from helpers import EPS, TOL, attn_std, rel_err, shape

SCHED = [212, 12]
L_S = 200


def _uniform(q, k, v, q_pos, n_heads):
    """Planted mistake: every visible key gets the same weight."""
    vis = np.arange(k.shape[0])[None, :] <= np.asarray(q_pos)[:, None]
    w = vis / vis.sum(axis=1, keepdims=True)
    return w @ np.asarray(v, dtype=np.float64)


def _leak_one(q, k, v, q_pos, n_heads, _orig=O.masked_attention):
    """Planted mistake: query i also sees key q_pos[i] + 1."""
    return _orig(q, k, v, np.minimum(np.asarray(q_pos) + 1, k.shape[0] - 1), n_heads)


def _all_own_keys(q, k, v, q_pos, n_heads, _orig=O.masked_attention):
    """Planted mistake (Stage II): every NS token sees all of its candidate's
    NS keys, the later ones included."""
    return _orig(q, k, v, np.full(len(q_pos), k.shape[0] - 1), n_heads)


def _errors(std, monkeypatch):
    sh = shape(n_layers=2)
    W = make_weights(sh, 7, "bf16", std=std)
    S = gen_normal(1, (L_S, sh.d), "bf16")
    NS = gen_normal(2, (sh.L_NS, sh.d), "bf16")
    X0 = np.concatenate([S, NS])[None]
    fwd = O.forward(X0, W, sh.L_NS, sh.n_heads, EPS, SCHED)
    kv = O.stage1(S, W, sh.L_NS, sh.n_heads, EPS, SCHED)
    s2 = O.stage2(kv, NS, W, sh.n_heads, EPS)
    out = {}
    for name, fn in (("uniform", _uniform), ("leak_one", _leak_one)):
        with monkeypatch.context() as mp:
            mp.setattr(O, "masked_attention", fn)
            out[name] = rel_err(O.forward(X0, W, sh.L_NS, sh.n_heads, EPS, SCHED), fwd)
    with monkeypatch.context() as mp:
        mp.setattr(O, "masked_attention", _all_own_keys)
        out["all_own_keys"] = rel_err(O.stage2(kv, NS, W, sh.n_heads, EPS), s2)
    return out


def test_planted_attention_mistakes_exceed_tolerance_at_attention_scale(monkeypatch):
    err = _errors(attn_std(256), monkeypatch)
    for name, e in err.items():
        assert e > 2 * TOL["bf16"], (name, e)


def test_planted_attention_mistakes_hide_at_small_weights(monkeypatch):
    """Why the attention-scale tests exist: at std 0.02 all three mistakes
    pass the bf16 bar."""
    err = _errors(0.02, monkeypatch)
    for name, e in err.items():
        assert e < TOL["bf16"], (name, e)
