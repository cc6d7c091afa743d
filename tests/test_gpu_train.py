"""The training step (forward keeping each layer's input, backward with each
layer recomputed from it) through the C ABI against the oracle's backward:
the output, the input gradient and every weight gradient, each within
max-abs-error / RMS <= 2e-2 (bf16 operands, float32 accumulation and
gradients) or 1e-4 (float32 mode).  Weights at std 1/sqrt(d), so attention
is far from uniform and its backward matters."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from onetrans_synth import gen_normal, linear_pyramid
from oracle import onetrans as O
from helpers import EPS, TOL, attn_std, build, rel_err, shape, tdt, to_dev, to_np

import unified_transformer_recommender_b200 as ot  # noqa: E402

GRAD_TOL = {"bf16": 2e-2, "fp32": 1e-4}
KEYS = ("g_attn", "g_ffn", "Wqkv_S", "Wqkv_NS", "Wo", "W1_S", "b1_S", "W2_S", "b2_S", "W1_NS", "b1_NS",
        "W2_NS", "b2_NS")


@pytest.fixture(autouse=True)
def _policy_reset():
    yield
    ot.onetrans_set_kernel_policy(0)
    assert ot.onetrans_device_status() == 0


def run_train(b, X0, dY):
    m, sh = b.model, b.shape
    B, L0, d = X0.shape
    grads = {k: [torch.full(np.shape(b.W[k][l]), float("nan"), dtype=torch.float32, device="cuda")
                 for l in range(sh.n_layers)] for k in KEYS}
    out = torch.full(dY.shape, float("nan"), dtype=torch.float32, device="cuda")
    dx0 = torch.full(X0.shape, float("nan"), dtype=torch.float32, device="cuda")
    ws = m.workspace(ot.OP_TRAIN, B, L0 - sh.L_NS)
    ot.onetrans_forward_backward(m, to_dev(X0, tdt(b.dtype)), to_dev(dY, torch.float32), out, dx0, grads, ws)
    torch.cuda.synchronize()
    return to_np(out), to_np(dx0), {k: [to_np(t) for t in v] for k, v in grads.items()}


@pytest.mark.parametrize("dtype,policy,d,pyr", [("bf16", 0, 256, True), ("bf16", 1, 256, True),
                                                ("fp32", 0, 256, True), ("bf16", 0, 256, False),
                                                ("fp32", 0, 32, False), ("bf16", 0, 384, True)])
def test_forward_backward_matches_oracle(dtype, policy, d, pyr):
    ot.onetrans_set_kernel_policy(policy)
    if d == 32:
        sh = shape(n_layers=2, d=32, H=2, dff=128, L_NS=4)
    elif d == 384:
        sh = shape(n_layers=2, d=384, dff=1536, L_NS=16)
    else:
        sh = shape(n_layers=2)
    L_S = 100
    sched = linear_pyramid(L_S + sh.L_NS, sh.L_NS, 2) if pyr else None
    b = build(sh, 250, dtype, pyramid=sched, std=attn_std(d))
    X0 = gen_normal(251, (2, L_S + sh.L_NS, sh.d), dtype)
    n_out = sched[-1] if pyr else L_S + sh.L_NS
    dY = gen_normal(252, (2, n_out, sh.d), "fp32")
    out, dx0, grads = run_train(b, X0, dY)
    Y, dX, dW = O.forward_backward(X0, b.W, sh.L_NS, sh.n_heads, EPS, sched, dY)
    assert rel_err(out, Y) <= TOL[dtype]
    errs = {"dx0": rel_err(dx0, dX)}
    for k in KEYS:
        for l in range(sh.n_layers):
            assert np.isfinite(grads[k][l]).all(), (k, l)
            errs[f"{k}[{l}]"] = rel_err(grads[k][l], dW[k][l])
    bad = {k: e for k, e in errs.items() if not e <= GRAD_TOL[dtype]}
    assert not bad, (bad, errs)
