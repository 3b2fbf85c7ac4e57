"""GPU parity at a large batch: 4096 stage-1 images (x 0.82 G elements,
offset_mask 1.39 G elements, byte offsets past 2^31), forward and backward,
checked against the oracle on sampled images (every image's result depends on
that image alone)."""
import numpy as np
import pytest
import torch

import oracle
import deformable_convolution_sparse_b200 as dcn
from deformable_convolution_sparse_b200.workloads import WORKLOADS, make_inputs_on

pytestmark = pytest.mark.gpu

N = 4096
SAMPLE = [0, 1, 2047, 4094, 4095]


@pytest.fixture(scope="module")
def big(cuda_device):
    w = WORKLOADS["stage1_f16"]
    x, om = make_inputs_on(cuda_device, N, w.H, w.W, w.C, w.G, w.K, w.Hout, w.Wout, "f16", w.offsets, w.masks,
                           seed=77)
    assert om.numel() > 2 ** 30 and om.numel() * om.element_size() > 2 ** 31
    yield w, x, om
    del x, om
    torch.cuda.empty_cache()


def test_forward_large_batch(big):
    w, x, om = big
    out = dcn.forward(x, om, **w.kwargs())
    torch.cuda.synchronize()
    for i in SAMPLE:
        ref = oracle.dcnv4_forward(x[i:i + 1].double().cpu().numpy(), om[i:i + 1].double().cpu().numpy(),
                                   **w.kwargs())
        got = out[i:i + 1].double().cpu().numpy()
        assert np.abs(got - ref).max() <= 4e-3 * np.abs(ref).max(), i
    del out


def test_backward_large_batch(big):
    w, x, om = big
    g = torch.Generator(device=x.device).manual_seed(78)
    go = torch.randn(x.shape, generator=g, device=x.device).half()
    gx, gom = dcn.backward(x, om, go, **w.kwargs())
    torch.cuda.synchronize()
    for i in SAMPLE:
        rgx, rgom = oracle.dcnv4_backward(x[i:i + 1].double().cpu().numpy(), om[i:i + 1].double().cpu().numpy(),
                                          go[i:i + 1].double().cpu().numpy(), **w.kwargs())
        for got, ref in ((gx[i:i + 1], rgx), (gom[i:i + 1], rgom)):
            g64 = got.double().cpu().numpy()
            assert np.abs(g64 - ref).max() <= 1e-5 * np.abs(ref).max(), i
    del gx, gom, go
