"""The allocation-free auto-split entry point, for callers that cannot
allocate device memory (a plugin whose host server owns every device byte,
or a serving loop where cudaMalloc would stall the device).  Through the C
ABI, on two calls in a row that share the library's fixed scratch array, it
must give bit for bit the tokens of the workspace entry point (both run the
same kernels with the same tiling), and those tokens must match the oracle's
auto-split within the bf16 tolerance of the other tests.  Collected last so
that a run stopping at the first failure has already run every other test."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from onetrans_synth import gen_normal
from oracle import onetrans as O
from helpers import TOL, build, rel_err, shape, stored_err, to_dev, to_np

import unified_transformer_recommender_b200 as ot  # noqa: E402


def test_static_scratch_autosplit_matches_workspace_entry_point():
    sh = shape(n_layers=1)
    b = build(sh, 301, "bf16")
    m = b.model
    for call, N in enumerate((1000, 2730)):      # 2730 rows fill the 16 MiB array at H = 3072
        feats_np = gen_normal(400 + call, (N, sh.ns_feat), "bf16")
        feats = to_dev(feats_np, torch.bfloat16)
        ref = torch.empty(N, sh.L_NS, sh.d, dtype=torch.bfloat16, device="cuda")
        ot.onetrans_tokenize_autosplit(m, feats, ref, m.workspace(ot.OP_AUTOSPLIT, N))
        got = torch.full((N, sh.L_NS, sh.d), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = torch.cuda.current_stream().cuda_stream
        status = ot.lib.onetrans_tokenize_autosplit_static(m.handle, feats.data_ptr(), N, got.data_ptr(), st)
        assert status == ot.OK
        torch.cuda.synchronize()
        assert torch.equal(got, ref), call
        rows = np.unique(np.r_[0, 1, N // 2, N - 1, np.random.default_rng(call).integers(0, N, 60)])
        want = O.autosplit(feats_np[rows], b.W, sh.L_NS)
        assert stored_err(to_np(got)[rows], want, "bf16") <= TOL["bf16"], call
    # one row past the array's capacity is refused before any launch
    too_many = 2731
    feats = torch.zeros(too_many, sh.ns_feat, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(too_many, sh.L_NS, sh.d, dtype=torch.bfloat16, device="cuda")
    assert ot.lib.onetrans_tokenize_autosplit_static(m.handle, feats.data_ptr(), too_many, out.data_ptr(),
                                                     None) == ot.ERR_CAPACITY
    assert ot.onetrans_device_status() == 0
