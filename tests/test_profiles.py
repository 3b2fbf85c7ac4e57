"""The ncu summaries under profiles/: every summary names its command and carries
well-formed machine-readable fields (the ones bench.py reads for
roofline.traffic), and its DRAM bytes are plausible for the workload: at least
the input bytes a launch must read once and no more than the algorithmic bytes
plus the fp32 gradients the backward writes. The forward may read x a second
time: a band's halo rows are fetched again by the CTA that takes the
neighbouring band one strip later, when the steps rotate over input sets
larger than L2 and the rows have been evicted in between."""
import glob
import os
import re

import pytest

from deformable_convolution_sparse_b200.workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ALL = sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md")))
# ncu summaries of a kernel launch, and measurement summaries of probes
PROFILES = [p for p in ALL if not os.path.basename(p).startswith("probe_")]
PROBES = [p for p in ALL if os.path.basename(p).startswith("probe_")]
E = {"f32": 4, "f16": 2, "bf16": 2}


def _fields(path):
    out = {}
    with open(path) as f:
        for line in f:
            if line.startswith("- ") and ":" in line:
                k, v = line[2:].split(":", 1)
                out[k.strip()] = v.strip().split("` ")[0].strip("`")
    return out


def test_there_is_a_summary_per_kernel_family():
    passes = {_fields(p).get("pass") for p in PROFILES}
    assert {"forward", "backward", "predictor"} <= passes


@pytest.mark.parametrize("path", PROFILES, ids=os.path.basename)
def test_summary_fields(path):
    f = _fields(path)
    text = open(path).read()
    assert "ncu " in text and "--clock-control none" in text, "the command that made it"
    assert f["workload"] in WORKLOADS
    assert f["pass"] in ("forward", "backward", "predictor")
    assert re.fullmatch(r"[0-9a-f]{64}", f["kernel_sources_sha256"])
    w = WORKLOADS[f["workload"]]
    e = E[w.dtype]
    dram = int(f["dram_bytes_per_launch"])
    x = w.N * w.H * w.W * w.C * e
    om = w.N * w.Hout * w.Wout * w.G * 3 * w.K * w.K * e
    out = w.N * w.Hout * w.Wout * w.C * e
    kind = f["pass"]
    if kind == "forward":
        lo, hi = x + om, x + om + out + x
    elif kind == "backward":
        lo, hi = x + om + out, x + om + out + (x + om) // e * 4
    else:  # predictor: y [pixels, C] read, records written
        lo, hi = w.N * w.Hout * w.Wout * w.C * e, w.N * w.Hout * w.Wout * w.C * e + om
    assert 0.99 * lo <= dram <= 1.01 * hi, (lo, dram, hi)


@pytest.mark.parametrize("path", PROBES, ids=os.path.basename)
def test_probe_summary_names_its_command_and_values(path):
    text = open(path).read()
    name = os.path.basename(path)[len("probe_"):-len(".md")]
    assert "python -c" in text and f"probe_{name}(" in text
    # the rate is the first numeric cell after a table row's label
    rates = [float(v) for v in re.findall(r"^\| [^|]+\| ([0-9.]+) \|", text, re.M)]
    assert len(rates) >= 2 and all(1.0 < r <= 128.5 for r in rates), rates


@pytest.mark.parametrize("path", ALL, ids=os.path.basename)
def test_summary_is_short_text(path):
    assert os.path.getsize(path) < 16 * 1024
