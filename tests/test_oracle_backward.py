"""Pins of the oracle's backward pass against things other than itself.

* torch.autograd in float64: the stack rebuilt from torch routines
  (rms_norm, scaled_dot_product_attention with the causal mask, gelu), its
  forward checked equal to the oracle's, its gradients taken by autograd;
  with and without the pyramid, with mixed S / NS weights.
* Central finite differences of the oracle's own forward along random
  directions of the input and of every weight kind.
* The pieces alone: RMSNorm, GELU-tanh and masked attention against autograd.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from onetrans_synth import ModelShape, gen_normal, make_weights
from oracle import onetrans as O

EPS = 1e-6
KEYS = O._GRAD_KEYS


def tiny(seed=3, n_layers=2, d=32, H=2, dff=64, L_NS=3):
    sh = ModelShape(n_layers=n_layers, d=d, n_heads=H, d_ff=dff, L_NS=L_NS, ns_feat=8, ns_hidden=8,
                    behavior_dims=(4,))
    return sh, make_weights(sh, seed, "fp32", std=0.2)    # scores far from uniform


def t64(a, grad=False):
    return torch.tensor(np.asarray(a, dtype=np.float64), requires_grad=grad)


def torch_stack(X0, Wt, L_NS, H, eps, schedule):
    """The block stack from torch routines (float64), per-row weights by
    concatenating the shared S set (expanded) and the per-token NS sets."""
    outs = []
    N = len(Wt["Wo"])
    for b in range(X0.shape[0]):
        x = X0[b]
        for l in range(N):
            L, d = x.shape
            Lq = L if schedule is None else schedule[l]
            nS, dh = L - L_NS, d // H
            h = F.rms_norm(x, (d,), Wt["g_attn"][l], eps)
            Wr = torch.cat([Wt["Wqkv_S"][l].expand(nS, 3 * d, d), Wt["Wqkv_NS"][l]], 0)
            qkv = torch.einsum("lod,ld->lo", Wr, h)
            q, k, v = qkv[L - Lq:, :d], qkv[:, d:2 * d], qkv[:, 2 * d:]
            pos = torch.arange(L - Lq, L)
            mask = torch.arange(L)[None, :] <= pos[:, None]
            a = F.scaled_dot_product_attention(q.view(Lq, H, dh).transpose(0, 1), k.view(L, H, dh).transpose(0, 1),
                                               v.view(L, H, dh).transpose(0, 1), attn_mask=mask)
            a = a.transpose(0, 1).reshape(Lq, d)
            x1 = x[L - Lq:] + a @ Wt["Wo"][l].T
            h2 = F.rms_norm(x1, (d,), Wt["g_ffn"][l], eps)
            nSq = Lq - L_NS
            W1 = torch.cat([Wt["W1_S"][l].expand(nSq, *Wt["W1_S"][l].shape), Wt["W1_NS"][l]], 0)
            b1 = torch.cat([Wt["b1_S"][l].expand(nSq, -1), Wt["b1_NS"][l]], 0)
            W2 = torch.cat([Wt["W2_S"][l].expand(nSq, *Wt["W2_S"][l].shape), Wt["W2_NS"][l]], 0)
            b2 = torch.cat([Wt["b2_S"][l].expand(nSq, -1), Wt["b2_NS"][l]], 0)
            z = F.gelu(torch.einsum("lfd,ld->lf", W1, h2) + b1, approximate="tanh")
            x = x1 + torch.einsum("ldf,lf->ld", W2, z) + b2
        outs.append(x)
    return torch.stack(outs)


@pytest.mark.parametrize("schedule", [None, [12, 3], [9, 3]])
def test_backward_matches_torch_autograd(schedule):
    sh, W = tiny()
    L_S = 13
    X0 = gen_normal(5, (2, L_S + sh.L_NS, sh.d), "fp32")
    Y, dX, dW = O.forward_backward(X0, W, sh.L_NS, sh.n_heads, EPS, schedule,
                                   gen_normal(6, (2, schedule[-1] if schedule else L_S + sh.L_NS, sh.d), "fp32"))
    dY = gen_normal(6, Y.shape, "fp32")
    Xt = t64(X0, True)
    Wt = {key: [t64(W[key][l], True) for l in range(sh.n_layers)] for key in KEYS}
    Yt = torch_stack(Xt, Wt, sh.L_NS, sh.n_heads, EPS, schedule)
    np.testing.assert_allclose(Yt.detach().numpy(), Y, rtol=1e-10, atol=1e-10)
    (Yt * t64(dY)).sum().backward()
    np.testing.assert_allclose(dX, Xt.grad.numpy(), rtol=1e-9, atol=1e-10)
    for key in KEYS:
        for l in range(sh.n_layers):
            np.testing.assert_allclose(dW[key][l], Wt[key][l].grad.numpy(), rtol=1e-9, atol=1e-10,
                                       err_msg=f"{key}[{l}]")


def test_backward_matches_finite_differences():
    sh, W = tiny(seed=11)
    L_S, sched = 10, [11, 3]
    X0 = gen_normal(7, (1, L_S + sh.L_NS, sh.d), "fp32").astype(np.float64)
    dY = gen_normal(8, (1, 3, sh.d), "fp32").astype(np.float64)
    _, dX, dW = O.forward_backward(X0, W, sh.L_NS, sh.n_heads, EPS, sched, dY)
    rng = np.random.default_rng(9)

    def loss(X, Wd):
        return float(np.sum(O.forward(X, Wd, sh.L_NS, sh.n_heads, EPS, sched) * dY))

    h = 1e-5
    u = rng.standard_normal(X0.shape)
    fd = (loss(X0 + h * u, W) - loss(X0 - h * u, W)) / (2 * h)
    assert abs(fd - np.sum(dX * u)) <= 1e-7 * (1 + abs(fd))
    for key in KEYS:
        for l in range(sh.n_layers):
            u = rng.standard_normal(np.shape(W[key][l]))
            Wp = {k: [np.asarray(a, np.float64) for a in v] if isinstance(v, list) else v for k, v in W.items()}
            Wm = {k: [np.asarray(a, np.float64) for a in v] if isinstance(v, list) else v for k, v in W.items()}
            Wp[key][l] = Wp[key][l] + h * u
            Wm[key][l] = Wm[key][l] - h * u
            fd = (loss(X0, Wp) - loss(X0, Wm)) / (2 * h)
            assert abs(fd - np.sum(dW[key][l] * u)) <= 1e-7 * (1 + abs(fd)), (key, l)


def test_rmsnorm_and_gelu_backward_match_autograd():
    x = gen_normal(10, (6, 16), "fp32")
    g = 1 + 0.1 * gen_normal(11, (16,), "fp32")
    dy = gen_normal(12, (6, 16), "fp32")
    xt, gt = t64(x, True), t64(g, True)
    (F.rms_norm(xt, (16,), gt, EPS) * t64(dy)).sum().backward()
    dx, dg = O.rmsnorm_backward(x, g, EPS, dy)
    np.testing.assert_allclose(dx, xt.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dg, gt.grad.numpy(), rtol=1e-11, atol=1e-12)
    u = np.linspace(-6, 6, 97)
    ut = t64(u, True)
    F.gelu(ut, approximate="tanh").sum().backward()
    np.testing.assert_allclose(O.gelu_tanh_grad(u), ut.grad.numpy(), rtol=1e-12, atol=1e-13)


def test_masked_attention_backward_matches_autograd():
    Lq, Lk, H, dh = 5, 9, 2, 4
    q = gen_normal(13, (Lq, H * dh), "fp32")
    k = gen_normal(14, (Lk, H * dh), "fp32")
    v = gen_normal(15, (Lk, H * dh), "fp32")
    do = gen_normal(16, (Lq, H * dh), "fp32")
    pos = np.arange(Lk - Lq, Lk)
    qt, kt, vt = t64(q, True), t64(k, True), t64(v, True)
    mask = torch.arange(Lk)[None, :] <= torch.as_tensor(pos)[:, None]
    o = F.scaled_dot_product_attention(qt.view(Lq, H, dh).transpose(0, 1), kt.view(Lk, H, dh).transpose(0, 1),
                                       vt.view(Lk, H, dh).transpose(0, 1), attn_mask=mask)
    (o.transpose(0, 1).reshape(Lq, -1) * t64(do)).sum().backward()
    dq, dk, dv = O.masked_attention_backward(q, k, v, pos, H, do)
    for a, b in ((dq, qt), (dk, kt), (dv, vt)):
        np.testing.assert_allclose(a, b.grad.numpy(), rtol=1e-10, atol=1e-12)
