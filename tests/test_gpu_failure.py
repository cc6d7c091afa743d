"""Failure path of the bounded waits, without faulting the GPU.  Every wait
of the tensor-core kernels is bounded: when it gives up it records a code in
the device status word and the kernel drains and returns instead of hanging.
Here a self-test kernel waits, with that same wait limited to a few rounds,
on an mbarrier that nothing arrives at: the call returns, the status word
reads the wait-timeout code (reported as ONETRANS_ERR_DEVICE_CHECK by the C
ABI) and is cleared by the read, and the context stays usable for a real
call afterwards."""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from onetrans_synth import gen_normal
from oracle import onetrans as O
from helpers import EPS, TOL, attn_std, build, rel_err, run_forward, shape

import unified_transformer_recommender_b200 as ot  # noqa: E402

WAIT_TIMEOUT = 101


def test_bounded_wait_runs_out_and_reports():
    assert ot.onetrans_device_status() == 0
    ot.onetrans_selftest_bounded_wait(64)
    code = ot.I32(-1)
    s = ot.lib.onetrans_device_status(torch.cuda.current_stream().cuda_stream, ctypes.byref(code))
    assert s == ot.ERR_DEVICE_CHECK and code.value == WAIT_TIMEOUT
    assert ot.onetrans_device_status() == 0           # the read cleared it
    # the context still runs the library's kernels correctly
    sh = shape(n_layers=1)
    b = build(sh, 240, "bf16", pyramid=[sh.L_NS], std=attn_std(sh.d))
    X0 = gen_normal(241, (2, 100 + sh.L_NS, sh.d), "bf16")
    got = run_forward(b, X0)
    assert ot.onetrans_device_status() == 0
    assert rel_err(got, O.forward(X0, b.W, sh.L_NS, sh.n_heads, EPS, [sh.L_NS])) <= TOL["bf16"]
