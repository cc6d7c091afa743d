"""Degenerate and boundary shapes of the method through the C ABI, against
the oracle: a merged sequence with no S token or a single one, a single NS
token, narrow heads (d_h = 16 and 32, which the tensor-core attention does
not take, so the CUDA-core kernels run beside the tensor-core GEMMs), and a
pyramid whose first layer already keeps only the NS rows.  Weights at std
1/sqrt(d) so that attention matters."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from onetrans_synth import gen_normal
from oracle import onetrans as O
from helpers import EPS, TOL, attn_std, build, rel_err, run_forward, run_stage12, shape

import unified_transformer_recommender_b200 as ot  # noqa: E402


@pytest.fixture(autouse=True)
def _status_clear():
    yield
    ot.onetrans_set_kernel_policy(0)
    assert ot.onetrans_device_status() == 0


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("L_S,pyr", [(0, False), (0, True), (1, False), (1, True), (130, "ns_only")])
def test_forward_short_and_ns_only_sequences(dtype, L_S, pyr):
    """No S token (the NS tokens attend to each other only), one S token, and
    a schedule whose first layer keeps only the NS rows."""
    sh = shape(n_layers=2)
    if pyr == "ns_only":
        sched = [sh.L_NS, sh.L_NS]
    else:
        sched = [L_S + sh.L_NS, sh.L_NS] if pyr else None
    b = build(sh, 270, dtype, pyramid=sched, std=attn_std(sh.d))
    X0 = gen_normal(271, (3, L_S + sh.L_NS, sh.d), dtype)
    got = run_forward(b, X0)
    ref = O.forward(X0, b.W, sh.L_NS, sh.n_heads, EPS, sched)
    assert got.shape == ref.shape
    assert rel_err(got, ref) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_single_ns_token(dtype):
    """L_NS = 1: one NS weight set, Stage II tiles of 128 candidates, each
    candidate's own key tile holding only its own key."""
    sched = [150 + 1, 40, 1]
    sh = shape(n_layers=3, L_NS=1, Hh=256)
    b = build(sh, 272, dtype, pyramid=sched, std=attn_std(sh.d))
    S = gen_normal(273, (2, 150, sh.d), dtype)
    NS = gen_normal(274, (300, 1, sh.d), dtype)
    _, out = run_stage12(b, S, NS, [0, 170, 300])
    X0 = np.concatenate([S[0], NS[0]])[None]
    assert rel_err(run_forward(b, X0)[0], O.forward(X0, b.W, 1, sh.n_heads, EPS, sched)[0]) <= TOL[dtype]
    for u, (c0, c1) in enumerate(((0, 170), (170, 300))):
        kv = O.stage1(S[u], b.W, 1, sh.n_heads, EPS, sched)
        for c in (c0, (c0 + c1) // 2, c1 - 1):
            assert rel_err(out[c], O.stage2(kv, NS[c], b.W, sh.n_heads, EPS)) <= TOL[dtype], (u, c)


@pytest.mark.parametrize("d,H", [(128, 4), (64, 4)])
def test_narrow_heads_mix_kernel_sets(d, H):
    """d_h = 32 and 16 in bf16: the attention runs on the CUDA-core kernels,
    the projections on the tensor-core GEMMs where their shapes allow."""
    sh = shape(n_layers=2, d=d, H=H, dff=4 * d)
    sched = [200 + sh.L_NS, sh.L_NS]
    b = build(sh, 275, "bf16", pyramid=sched, std=attn_std(d))
    S = gen_normal(276, (2, 200, d), "bf16")
    NS = gen_normal(277, (25, sh.L_NS, d), "bf16")
    _, out = run_stage12(b, S, NS, [0, 11, 25])
    for u, (c0, c1) in enumerate(((0, 11), (11, 25))):
        kv = O.stage1(S[u], b.W, sh.L_NS, sh.n_heads, EPS, sched)
        for c in range(c0, c1):
            assert rel_err(out[c], O.stage2(kv, NS[c], b.W, sh.n_heads, EPS)) <= TOL["bf16"], (u, c)
