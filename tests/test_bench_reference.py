"""The benchmark's reference arm (the fp64 oracle timed on the host cores) on
CPU: for every workload it prints one JSON line that names the same metric,
unit and config as the CUDA arm's line, with its CPU-baseline and
end-to-end objects."""
import json
import os
import subprocess
import sys
import types

import pytest

import bench
from onetrans_synth import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("workload", ["kv_serving", "append", "s_forward", "l_forward", "train"])
def test_reference_line_names_the_workload_of_the_cuda_arm(workload):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--workload", workload],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    metric, unit, config, units = bench.workload_meta(workload, 1)
    assert line["impl"] == "reference"
    assert (line["metric"], line["unit"], line["config"]) == (metric, unit, config)
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["ms_per_step"] == pytest.approx(1e3 * units / line["value"])
    assert line["dtype"] == "f64" and line["data"] == "synthetic"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["unit"] == unit
    assert cb["cores"] >= 1 and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": unit, "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_workload_classes_describe_themselves_as_the_shared_descriptions():
    """At the default sizes, the CUDA arm's workload objects report the
    metric, unit and config the reference arm prints."""
    for ws in (1, 4):
        kv, ap = WORKLOADS["kv_serving"], WORKLOADS["append"]
        m, u, c, _ = bench.workload_meta("kv_serving", ws)
        assert (bench.KVServing.metric, bench.KVServing.unit) == (m, u)
        assert bench.KVServing.config(types.SimpleNamespace(U=kv.users, C=kv.cands), ws) == c
        m, u, c, _ = bench.workload_meta("append", ws)
        assert (bench.Append.metric, bench.Append.unit) == (m, u)
        assert bench.Append.config(types.SimpleNamespace(U=ap.users, C=ap.cands, dL=ap.dL), ws) == c
        for name in ("s_forward", "l_forward"):
            m, u, c, _ = bench.workload_meta(name, ws)
            assert bench.Forward.unit == u
            assert bench.Forward.config(types.SimpleNamespace(name=name, U=WORKLOADS[name].users), ws) == c


def test_reference_arm_on_other_ranks_does_no_work(capsys):
    args = types.SimpleNamespace(workload="kv_serving", gpus=2, steps=1, warmup=0)
    assert bench.run_reference(args, rank=1) is None
    assert capsys.readouterr().out == ""
