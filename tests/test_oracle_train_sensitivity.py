"""The training step's gradient bar can see backward mistakes.

Mistakes are planted in the oracle's backward, on the CPU: the RMSNorm
backward without its mean term (the r^3 x sum(g dy x)/d part), the softmax
backward without its row term D = rowsum(dP P), and the GELU derivative
without its second term.  Each moves some gradient of the stack by more
than twice the norm-wise bf16 bar of `test_gpu_train.py`
(||got - ref|| / ||ref|| <= 2e-2; on these inputs by 0.27, 1.36 and 0.37),
so a kernel with that mistake fails it, while bf16 rounding of the operands
costs about 5e-3 norm-wise (the bar's derivation).  Weights at std 1/sqrt(d), as in the GPU training tests."""
import numpy as np
import pytest

from onetrans_synth import gen_normal, linear_pyramid, make_weights
from oracle import onetrans as O
from helpers import EPS, attn_std, shape

BAR = 2e-2


def _rms_no_mean(x, g, eps, dy, _orig=O.rmsnorm_backward):
    """Planted mistake: dx = r g dy (the mean term dropped)."""
    x64, g64, dy64 = (np.asarray(t, dtype=np.float64) for t in (x, g, dy))
    r = 1.0 / np.sqrt(np.mean(x64 * x64, axis=-1, keepdims=True) + eps)
    _, dg = _orig(x, g, eps, dy)
    return r * dy64 * g64, dg


def _attn_no_rowterm(q, k, v, q_pos, n_heads, do):
    """Planted mistake: dS = P dP (the row term D left out)."""
    q, k, v, do = (np.asarray(t, dtype=np.float64) for t in (q, k, v, do))
    Lq, d = q.shape
    dh = d // n_heads
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    visible = np.arange(k.shape[0])[None, :] <= np.asarray(q_pos)[:, None]
    for h in range(n_heads):
        sl = slice(h * dh, (h + 1) * dh)
        s = np.where(visible, q[:, sl] @ k[:, sl].T / np.sqrt(dh), -np.inf)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        dv[:, sl] = p.T @ do[:, sl]
        ds = p * (do[:, sl] @ v[:, sl].T)
        dq[:, sl] = ds @ k[:, sl] / np.sqrt(dh)
        dk[:, sl] = ds.T @ q[:, sl] / np.sqrt(dh)
    return dq, dk, dv


def _gelu_grad_first_term(x):
    """Planted mistake: GELU'(u) = 0.5 (1 + tanh(v)) only."""
    x = np.asarray(x, dtype=np.float64)
    c = np.sqrt(2.0 / np.pi)
    return 0.5 * (1.0 + np.tanh(c * (x + 0.044715 * x ** 3)))


def _worst_error(ref, got):
    """Largest norm-wise error over dX0 and every weight gradient."""
    _, dX_r, dW_r = ref
    _, dX_g, dW_g = got
    errs = [np.linalg.norm(dX_g - dX_r) / np.linalg.norm(dX_r)]
    for key in dW_r:
        for l in range(len(dW_r[key])):
            n = np.linalg.norm(dW_r[key][l])
            if n > 0:
                errs.append(np.linalg.norm(dW_g[key][l] - dW_r[key][l]) / n)
    return max(errs)


@pytest.mark.parametrize("name,attr,fn", [("rmsnorm mean term", "rmsnorm_backward", _rms_no_mean),
                                          ("softmax row term", "masked_attention_backward", _attn_no_rowterm),
                                          ("GELU second term", "gelu_tanh_grad", _gelu_grad_first_term)])
def test_planted_backward_mistakes_exceed_the_gradient_bar(name, attr, fn, monkeypatch):
    sh = shape(n_layers=2, d=64, H=4, dff=256, L_NS=4)
    L_S = 40
    sched = linear_pyramid(L_S + sh.L_NS, sh.L_NS, 2)
    W = make_weights(sh, 31, "bf16", std=attn_std(sh.d))
    X0 = gen_normal(32, (2, L_S + sh.L_NS, sh.d), "bf16")
    dY = gen_normal(33, (2, sched[-1], sh.d), "fp32")
    ref = O.forward_backward(X0, W, sh.L_NS, sh.n_heads, EPS, sched, dY)
    with monkeypatch.context() as mp:
        mp.setattr(O, attr, fn)
        got = O.forward_backward(X0, W, sh.L_NS, sh.n_heads, EPS, sched, dY)
    err = _worst_error(ref, got)
    assert err > 2 * BAR, (name, err)
