"""The benchmark's reference arm (the fp64 oracle on the host cores) on CPU: one
JSON line with the contract's keys, the same metric, unit and workload text as
this implementation's line for the same pass and variant, and no output from
ranks other than 0."""
import json
import os
import subprocess
import sys

import pytest

import bench
from deformable_convolution_sparse_b200.workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
        "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"}


def _run(*args, env=None):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny_f32",
           "--steps", "2", "--warmup", "1", *args]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    return r.stdout


@pytest.mark.parametrize("which,variant", [("forward", "none"), ("forward", "all"), ("backward", "none"),
                                           ("backward", "softmax"), ("predictor", "none")])
def test_reference_line(which, variant):
    out = _run("--pass", which, "--variant", variant)
    lines = [ln for ln in out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert KEYS <= set(d)
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 2 and d["warmup"] == 1
    metric = {"forward": bench.METRIC, "backward": bench.METRIC_BWD, "predictor": bench.METRIC_PRED}[which]
    unit = "Grecords/s" if which == "predictor" else bench.UNIT
    assert d["metric"] == metric and d["unit"] == unit
    assert d["config"]["workload"] == bench.workload_text(WORKLOADS["tiny_f32"], which, variant)
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d.get("pass") == (None if which == "forward" else which)


def test_other_ranks_print_nothing():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    assert _run(env=env).strip() == ""


def test_workload_text_names_each_shape():
    assert "stage-1" in bench.workload_text(WORKLOADS["stage1_f16"])
    assert "stage-3" in bench.workload_text(WORKLOADS["stage3_f16"])
    assert "SD-1.5" in bench.workload_text(WORKLOADS["sd_latent_f16"])
    assert "dilation=2" in bench.workload_text(WORKLOADS["highres_bf16"])
    assert "8 points per unit" in bench.workload_text(WORKLOADS["stage1_f16"], "forward", "remove_center")
