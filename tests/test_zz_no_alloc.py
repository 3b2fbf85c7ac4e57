"""GPU test of dcnv4_forward_host_noalloc, the entry point for callers that
cannot allocate device memory when they call the library (for example a
serving process whose GPU memory already belongs to its own pool, or a
latency-critical path where cudaMalloc/cudaFree could synchronise the device).
It stages through the library's fixed device array instead of caller buffers.

The file is named so that pytest collects it last. It must pass on its own in
a fresh process (the first call sets up the array's device address) and after
every other test.
"""
import ctypes

import pytest
import torch

import deformable_convolution_sparse_b200 as dcn
from deformable_convolution_sparse_b200.workloads import WORKLOADS, make_inputs, workload_inputs

pytestmark = pytest.mark.gpu


def _noalloc_via_c_abi(x, om, out, w):
    """One call of the C entry point with host pointers only, then wait."""
    lib = dcn.load_library()
    stream = torch.cuda.current_stream()
    rc = lib.dcnv4_forward_host_noalloc(x.data_ptr(), om.data_ptr(), out.data_ptr(), w.N, w.H, w.W, w.C, w.G, w.K,
                                        w.stride, w.pad, w.dilation, ctypes.c_float(w.offset_scale),
                                        dcn.binding.TORCH_DTYPE[x.dtype], stream.cuda_stream)
    assert rc == dcn.DCNV4_OK, dcn.strerror(rc)
    stream.synchronize()


def test_noalloc_matches_host_path_on_two_calls_in_a_row(cuda_device):
    torch.cuda.set_device(cuda_device)
    # two different problems back to back: the second call must not see the first one's data
    first = WORKLOADS["stage1_f16"]
    second = WORKLOADS["stage1_f16"].with_(seed=77)
    for w in (first, second):
        x, om = workload_inputs(w)
        x, om = x.pin_memory(), om.pin_memory()
        out = torch.full((w.N, w.Hout, w.Wout, w.C), float("nan"), dtype=x.dtype).pin_memory()
        _noalloc_via_c_abi(x, om, out, w)
        ref = dcn.forward_host(x, om, device=cuda_device, **w.kwargs())
        # the same kernels on the same inputs: equal within the fp16 tolerance
        scale = ref.double().abs().max().item()
        err = (out.double() - ref.double()).abs().max().item()
        assert err <= 4e-3 * scale, (w.seed, err, scale)
        assert not torch.isnan(out).any()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_noalloc_other_dtypes_and_many_chunks(dtype, cuda_device):
    # 40 images of 96x96x64 need several chunks of the 16 MiB staging halves
    N, H, W, C, G, K = 40, 96, 96, 64, 4, 3
    x, om = make_inputs(N, H, W, C, G, K, H, W, dtype, ("normal", 0, 1.5), ("normal", 0, 0.5), seed=5)
    out = dcn.forward_host_noalloc(x.pin_memory(), om.pin_memory(), G=G, K=K, pad=1)
    ref = dcn.forward(x.to(cuda_device), om.to(cuda_device), G=G, K=K, pad=1).cpu()
    tol = 1e-5 if dtype == "f32" else 4e-3
    scale = ref.double().abs().max().item()
    assert (out.double() - ref.double()).abs().max().item() <= tol * scale


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
