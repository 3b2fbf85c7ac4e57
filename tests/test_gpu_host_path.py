"""GPU tests of dcnv4_forward_host: inputs and result in host memory, the
device buffers only as staging, the copies and kernels pipelined over image
chunks. The result must equal the device-resident forward bit for bit."""
import os
import re
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
import deformable_convolution_sparse_b200 as dcn
from deformable_convolution_sparse_b200.workloads import WORKLOADS, make_inputs, workload_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("pinned", [True, False])
@pytest.mark.parametrize("N", [1, 3, 8, 11])
def test_host_path_equals_device_path(N, pinned, cuda_device):
    x, om = make_inputs(N, 17, 19, 64, 4, 3, 17, 19, "f16", ("normal", 0, 1.5), ("normal", 0, 0.5), seed=N)
    if pinned:
        x, om = x.pin_memory(), om.pin_memory()
    out = dcn.forward_host(x, om, G=4, K=3, pad=1, device=cuda_device)
    ref = dcn.forward(x.to(cuda_device), om.to(cuda_device), G=4, K=3, pad=1).cpu()
    assert torch.equal(out, ref)


@pytest.mark.parametrize("chunks", [None, "7", "1"])
def test_host_path_chunkings_equal_device_path(chunks, cuda_device, monkeypatch):
    # 45 stage-1 sized images (results smaller than their records: x goes over in one copy ahead
    # of the records' chunks): the library's own chunking, 7 uneven chunks and a single chunk
    if chunks is not None:
        monkeypatch.setenv("DCNV4_HOST_CHUNKS", chunks)
    x, om = make_inputs(45, 56, 56, 64, 4, 3, 56, 56, "f16", ("normal", 0, 1.5), ("normal", 0, 0.5), seed=45)
    out = dcn.forward_host(x.pin_memory(), om.pin_memory(), G=4, K=3, pad=1, device=cuda_device)
    ref = dcn.forward(x.to(cuda_device), om.to(cuda_device), G=4, K=3, pad=1).cpu()
    assert torch.equal(out, ref)


@pytest.mark.parametrize("chunks", [None, "5"])
def test_host_path_results_larger_than_records_equal_device_path(chunks, cuda_device, monkeypatch):
    # C = 256 channels in 4 groups: a result pixel (512 B) outweighs its records (216 B), so each
    # chunk carries its own x and offset_mask
    if chunks is not None:
        monkeypatch.setenv("DCNV4_HOST_CHUNKS", chunks)
    x, om = make_inputs(13, 40, 40, 256, 4, 3, 40, 40, "f16", ("normal", 0, 1.5), ("normal", 0, 0.5), seed=13)
    out = dcn.forward_host(x.pin_memory(), om.pin_memory(), G=4, K=3, pad=1, device=cuda_device)
    ref = dcn.forward(x.to(cuda_device), om.to(cuda_device), G=4, K=3, pad=1).cpu()
    assert torch.equal(out, ref)


# Fewer images than chunks: each image is cut into bands of output rows, one launch per band over
# the whole image (unit windows, image windows, the global-gather kernel, stride 2, dilation 2,
# one-row bands, bands too short for the whole image's item size)
BAND_CASES = [
    # N, H, W, C, G, K, stride, pad, dilation, dtype, chunks
    (2, 64, 64, 128, 8, 3, 1, 2, 2, "bf16", "8"),
    (1, 56, 56, 64, 4, 3, 1, 1, 1, "f16", "5"),
    (1, 14, 14, 256, 16, 3, 1, 1, 1, "f16", "3"),
    (1, 20, 20, 48, 2, 3, 1, 1, 1, "f16", "4"),
    (3, 33, 29, 64, 4, 3, 2, 1, 1, "f32", "7"),
    (1, 9, 9, 32, 2, 3, 1, 1, 1, "f32", "64"),
    (2, 32, 32, 256, 4, 3, 1, 1, 1, "f16", "6"),  # results larger than records: x with each first band
    (1, 9, 9, 32, 1, 3, 1, 1, 1, "f16", "3"),  # a band's records start 2-byte aligned (486-byte rows)
]


@pytest.mark.parametrize("case", BAND_CASES)
def test_host_path_row_bands_equal_device_path(case, cuda_device, monkeypatch):
    N, H, W, C, G, K, s, pad, d, dtype, chunks = case
    monkeypatch.setenv("DCNV4_HOST_CHUNKS", chunks)
    Ho = (H + 2 * pad - d * (K - 1) - 1) // s + 1
    Wo = (W + 2 * pad - d * (K - 1) - 1) // s + 1
    x, om = make_inputs(N, H, W, C, G, K, Ho, Wo, dtype, ("normal", 0, 2.0), ("normal", 0, 0.5), seed=H + N)
    kw = dict(G=G, K=K, stride=s, pad=pad, dilation=d)
    out = dcn.forward_host(x.pin_memory(), om.pin_memory(), device=cuda_device, **kw)
    ref = dcn.forward(x.to(cuda_device), om.to(cuda_device), **kw).cpu()
    assert torch.equal(out, ref)


def test_host_path_planner_override_keeps_the_device_result(cuda_device, monkeypatch):
    # an item height forced above the bands' row counts leaves the bands without a ring plan of the
    # image's kind: the host path must then keep whole images (same bits as the device path)
    monkeypatch.setenv("DCNV4_HOST_CHUNKS", "8")
    monkeypatch.setenv("DCNV4_TILE", "14x14")
    x, om = make_inputs(2, 28, 28, 64, 4, 3, 28, 28, "f16", ("normal", 0, 1.5), ("normal", 0, 0.5), seed=11)
    out = dcn.forward_host(x.pin_memory(), om.pin_memory(), G=4, K=3, pad=1, device=cuda_device)
    ref = dcn.forward(x.to(cuda_device), om.to(cuda_device), G=4, K=3, pad=1).cpu()
    assert torch.equal(out, ref)


def test_host_path_row_bands_from_pageable_memory(cuda_device, monkeypatch):
    # pageable host buffers: the copies block the calling thread, the bands and their order stay
    monkeypatch.setenv("DCNV4_HOST_CHUNKS", "6")
    x, om = make_inputs(2, 40, 40, 64, 4, 3, 40, 40, "f16", ("normal", 0, 2.0), ("normal", 0, 0.5), seed=9)
    out = dcn.forward_host(x, om, G=4, K=3, pad=1, device=cuda_device)
    ref = dcn.forward(x.to(cuda_device), om.to(cuda_device), G=4, K=3, pad=1).cpu()
    assert torch.equal(out, ref)


_BANDS_RUN = r"""
import sys, torch
sys.path.insert(0, sys.argv[1])
import deformable_convolution_sparse_b200 as dcn
from deformable_convolution_sparse_b200.workloads import make_inputs
x, om = make_inputs(2, 64, 64, 128, 8, 3, 62, 62, "bf16", ("normal", 0, 2.0), ("normal", 0, 0.5), seed=5)
dcn.forward_host(x.pin_memory(), om.pin_memory(), G=8, K=3, pad=1, dilation=2, device=torch.device("cuda:0"))
torch.cuda.synchronize()
"""


def test_host_path_launches_one_plan_per_band(cuda_device):
    # two images in eight chunks: four bands of 15-16 output rows per image, each its own launch
    # (DCNV4_DEBUG=1 prints the ring plan of every launch); the whole-image schedule would make two
    env = dict(os.environ, DCNV4_DEBUG="1", DCNV4_HOST_CHUNKS="8")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = subprocess.run([sys.executable, "-c", _BANDS_RUN, root], capture_output=True, text=True, timeout=300,
                         env=env)
    assert res.returncode == 0, res.stderr[-2000:]
    plans = re.findall(r"dcnv4 ring plan: .* rows_total (\d+)", res.stderr)
    assert len(plans) == 8, res.stderr[-2000:]


def test_host_path_full_workload_against_oracle(cuda_device):
    w = WORKLOADS["stage1_f16"]
    x, om = workload_inputs(w)
    out = dcn.forward_host(x.pin_memory(), om.pin_memory(), device=cuda_device, **w.kwargs())
    ref = oracle.dcnv4_forward(x.double().numpy(), om.double().numpy(), **w.kwargs())
    err = np.abs(out.double().numpy() - ref).max()
    assert err <= 4e-3 * np.abs(ref).max()


def test_host_path_reuses_caller_staging_and_orders_after_stream_work(cuda_device):
    x, om = make_inputs(4, 9, 9, 32, 2, 3, 9, 9, "f32", seed=3)
    staging = (torch.full_like(x, 7.0, device=cuda_device), torch.full_like(om, 7.0, device=cuda_device),
               torch.full((4, 9, 9, 32), 7.0, device=cuda_device))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        torch.cuda._sleep(1_000_000)  # queued work the call must come after
        out = dcn.forward_host(x.pin_memory(), om.pin_memory(), G=2, K=3, pad=1, staging=staging, stream=s)
    ref = oracle.dcnv4_forward(x.double().numpy(), om.double().numpy(), G=2, K=3, pad=1)
    assert np.abs(out.double().numpy() - ref).max() <= 1e-5 * np.abs(ref).max()
    assert torch.equal(staging[0].cpu(), x) and torch.equal(staging[2].cpu(), out)


def test_host_path_rejects_bad_arguments(cuda_device):
    lib = dcn.load_library()
    x = torch.zeros(2, 8, 8, 16).pin_memory()
    om = torch.zeros(2, 8, 8, 2, 27).pin_memory()
    out = torch.zeros(2, 8, 8, 16).pin_memory()
    xd, omd, od = x.to(cuda_device), om.to(cuda_device), out.to(cuda_device)
    args = (2, 8, 8, 16, 2, 3, 1, 1, 1, 1.0, 0, None)
    assert lib.dcnv4_forward_host(0, om.data_ptr(), out.data_ptr(), xd.data_ptr(), omd.data_ptr(), od.data_ptr(),
                                  *args) == dcn.STATUS["DCNV4_ERR_NULL"]
    assert lib.dcnv4_forward_host(x.data_ptr(), om.data_ptr(), x.data_ptr(), xd.data_ptr(), omd.data_ptr(),
                                  od.data_ptr(), *args) == dcn.STATUS["DCNV4_ERR_ALIAS"]
    assert lib.dcnv4_forward_host(x.data_ptr(), om.data_ptr(), out.data_ptr(), xd.data_ptr(), omd.data_ptr(),
                                  xd.data_ptr(), *args) == dcn.STATUS["DCNV4_ERR_ALIAS"]
