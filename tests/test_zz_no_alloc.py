"""GPU test of dcnv4_forward_host_noalloc, the entry point for callers that
cannot allocate device memory when they call the library (for example a
serving process whose GPU memory already belongs to its own pool, or a
latency-critical path where cudaMalloc/cudaFree could synchronise the device).
It stages through the library's fixed device array instead of caller buffers.

The forward's plan and arithmetic do not depend on the batch it is given, so
the chunks the entry point runs must give exactly the bits of one device-side
call over the whole batch: every comparison below is bit for bit.

The file is named so that pytest collects it last. It passes on its own in a
fresh process (the first call there looks up the array's device address,
which one test checks in a subprocess) and after every other test.
"""
import ctypes
import os
import subprocess
import sys

import pytest
import torch

import deformable_convolution_sparse_b200 as dcn
from deformable_convolution_sparse_b200.workloads import WORKLOADS, make_inputs, workload_inputs

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _noalloc_via_c_abi(x, om, out, w):
    """One call of the C entry point with host pointers only, then wait."""
    lib = dcn.load_library()
    stream = torch.cuda.current_stream()
    rc = lib.dcnv4_forward_host_noalloc(x.data_ptr(), om.data_ptr(), out.data_ptr(), w.N, w.H, w.W, w.C, w.G, w.K,
                                        w.stride, w.pad, w.dilation, ctypes.c_float(w.offset_scale),
                                        dcn.binding.TORCH_DTYPE[x.dtype], stream.cuda_stream)
    assert rc == dcn.DCNV4_OK, dcn.strerror(rc)
    stream.synchronize()


def test_noalloc_matches_the_device_forward_on_two_calls_in_a_row(cuda_device):
    torch.cuda.set_device(cuda_device)
    # two different problems back to back: the second call must not see the first one's data
    first = WORKLOADS["stage1_f16"]
    second = WORKLOADS["stage1_f16"].with_(seed=77)
    for w in (first, second):
        x, om = workload_inputs(w)
        x, om = x.pin_memory(), om.pin_memory()
        out = torch.full((w.N, w.Hout, w.Wout, w.C), float("nan"), dtype=x.dtype).pin_memory()
        _noalloc_via_c_abi(x, om, out, w)
        ref = dcn.forward(x.to(cuda_device), om.to(cuda_device), **w.kwargs()).cpu()
        assert torch.equal(out, ref), w.seed


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_noalloc_other_dtypes_and_many_chunks(dtype, cuda_device):
    # 40 images of 96x96x64 need several chunks of the 16 MiB staging halves
    N, H, W, C, G, K = 40, 96, 96, 64, 4, 3
    x, om = make_inputs(N, H, W, C, G, K, H, W, dtype, ("normal", 0, 1.5), ("normal", 0, 0.5), seed=5)
    out = dcn.forward_host_noalloc(x.pin_memory(), om.pin_memory(), G=G, K=K, pad=1)
    ref = dcn.forward(x.to(cuda_device), om.to(cuda_device), G=G, K=K, pad=1).cpu()
    assert torch.equal(out, ref)


def test_noalloc_with_pageable_host_memory(cuda_device):
    """Unpinned host buffers: the copies then block the calling thread, and the
    result must be the same bits."""
    N, H, W, C, G, K = 12, 64, 64, 64, 4, 3
    x, om = make_inputs(N, H, W, C, G, K, H, W, "f16", ("normal", 0, 1.5), ("normal", 0, 0.5), seed=8)
    assert not x.is_pinned() and not om.is_pinned()
    out = torch.empty((N, H, W, C), dtype=x.dtype)
    w = WORKLOADS["stage1_f16"].with_(N=N, H=H, W=W, Hout=H, Wout=W)
    _noalloc_via_c_abi(x, om, out, w)
    ref = dcn.forward(x.to(cuda_device), om.to(cuda_device), G=G, K=K, pad=1).cpu()
    assert torch.equal(out, ref)


_FRESH = r"""
import ctypes, sys, torch
sys.path.insert(0, sys.argv[1])
import deformable_convolution_sparse_b200 as dcn
from deformable_convolution_sparse_b200.workloads import make_inputs
x, om = make_inputs(3, 40, 44, 64, 4, 3, 40, 44, "f16", ("normal", 0, 2.0), ("normal", 0, 0.5), seed=19)
x, om = x.pin_memory(), om.pin_memory()
out = torch.empty((3, 40, 44, 64), dtype=x.dtype).pin_memory()
lib = dcn.load_library()
# the very first call of the library in this process: it looks up the array's device address
rc = lib.dcnv4_forward_host_noalloc(x.data_ptr(), om.data_ptr(), out.data_ptr(), 3, 40, 44, 64, 4, 3, 1, 1, 1,
                                    ctypes.c_float(1.0), dcn.DCNV4_F16, None)
torch.cuda.synchronize()
assert rc == 0, dcn.strerror(rc)
ref = dcn.forward(x.cuda(), om.cuda(), G=4, K=3, pad=1).cpu()
assert torch.equal(out, ref)
print("fresh-process noalloc ok")
"""


def test_noalloc_as_the_first_call_of_a_fresh_process(cuda_device):
    res = subprocess.run([sys.executable, "-c", _FRESH, ROOT], capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "fresh-process noalloc ok" in res.stdout


def test_noalloc_rejects_an_image_beyond_the_staging_area(cuda_device):
    lib = dcn.load_library()
    # one 300x300x64 fp32 image: x + offset_mask + out ~ 82 MB > 16 MiB, rejected before any copy
    x = torch.zeros(1, 300, 300, 64)
    om = torch.zeros(1, 300, 300, 4, 27)
    out = torch.zeros(1, 300, 300, 64)
    rc = lib.dcnv4_forward_host_noalloc(x.data_ptr(), om.data_ptr(), out.data_ptr(), 1, 300, 300, 64, 4, 3, 1, 1, 1,
                                        ctypes.c_float(1.0), dcn.DCNV4_F32, None)
    assert rc == dcn.STATUS["DCNV4_ERR_STAGING"]
    assert "staging" in dcn.strerror(rc)
