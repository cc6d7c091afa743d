"""The training step (forward keeping each layer's input, attention output and
log-sum-exp; backward with the rest of each layer recomputed) through the C
ABI against the oracle's backward (which recomputes whole layers; the
gradients are the same):
the output, the input gradient and every weight gradient.  Weights at std
1/sqrt(d), so attention is far from uniform and its backward matters.

Bars.  Float32 mode: max-abs-error / RMS <= 1e-4 for every tensor, element
by element.  BF16 mode (bf16 operands of every contraction, float32
accumulation and gradients): the output within max-abs-error / RMS <= 2e-2
like the forward; the gradients within ||got - ref|| / ||ref|| <= 2e-2.  A
gradient that sums only a few rows (an NS set's weights sum one row per
sample) keeps the rounding of its two bf16 operands element by element, up
to 0.14 of the RMS on these inputs in a CPU emulation of exactly those
rounding points, while the norm-wise error stays near 5e-3; a dropped term
or a wrong row still moves it well past 2e-2.  A gradient whose reference
is exactly zero (the S set of a layer that keeps only NS rows) must be zero."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from onetrans_synth import gen_normal, linear_pyramid
from oracle import onetrans as O
from helpers import EPS, TOL, attn_std, build, rel_err, shape, tdt, to_dev, to_np

import unified_transformer_recommender_b200 as ot  # noqa: E402

def grad_err(got, ref, dtype) -> float:
    """fp32: max-abs-error / RMS; bf16: ||got - ref|| / ||ref||."""
    if dtype == "fp32":
        return rel_err(got, ref)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(np.asarray(got, dtype=np.float64) - ref) / np.linalg.norm(ref))


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


def check_train(dtype, sh, B, L_S, pyr, seed):
    sched = linear_pyramid(L_S + sh.L_NS, sh.L_NS, sh.n_layers) if pyr else None
    b = build(sh, seed, dtype, pyramid=sched, std=attn_std(sh.d))
    X0 = gen_normal(seed + 1, (B, L_S + sh.L_NS, sh.d), dtype)
    n_out = sched[-1] if pyr else L_S + sh.L_NS
    dY = gen_normal(seed + 2, (B, n_out, sh.d), "fp32")
    out, dx0, grads = run_train(b, X0, dY)
    Y, dX, dW = O.forward_backward(X0, b.W, sh.L_NS, sh.n_heads, EPS, sched, dY)
    assert rel_err(out, Y) <= TOL[dtype]
    errs = {"dx0": grad_err(dx0, dX, dtype)}
    for k in KEYS:
        for l in range(sh.n_layers):
            assert np.isfinite(grads[k][l]).all(), (k, l)
            if not np.any(dW[k][l]):
                assert not np.any(grads[k][l]), (k, l)
                continue
            errs[f"{k}[{l}]"] = grad_err(grads[k][l], dW[k][l], dtype)
    bad = {k: e for k, e in errs.items() if not e <= TOL[dtype]}
    assert not bad, (bad, errs)


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
    check_train(dtype, sh, 2, 100, pyr, 250)


def test_forward_backward_many_samples():
    """66 samples of 70 S tokens: the weight gradients' row tiles span
    several samples, the S set splits into many slices (partial gradients
    added afterwards) and each NS set's rows (one per sample) fill one tile of
    64 and part of a second."""
    check_train("bf16", shape(n_layers=2, dff=512), 66, 70, False, 253)
