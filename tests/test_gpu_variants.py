"""GPU parity of the forward variants (dcnv4_forward_ex through the C ABI:
DCNv3 softmax over the masks, centre point removed, centre feature scaling,
and all three together) against the oracle's variants, on every kernel path,
with the forward's bars: max|err| <= 1e-5 * max|out| for fp32 storage and
<= 4e-3 * max|out| for fp16/bf16."""
import numpy as np
import pytest
import torch

import oracle
import deformable_convolution_sparse_b200 as dcn
from deformable_convolution_sparse_b200.workloads import WORKLOADS, make_center_logit, make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "f16": 4e-3, "bf16": 4e-3}
VARIANTS = {
    "softmax": dict(softmax=True),
    "remove_center": dict(remove_center=True),
    "center_scale": dict(center=True),
    "all": dict(softmax=True, remove_center=True, center=True),
}


@pytest.fixture(params=["window", "window_unit", "window_f16exact", "gather"])
def variant(request, monkeypatch):
    monkeypatch.delenv("DCNV4_VARIANT", raising=False)
    monkeypatch.delenv("DCNV4_F16_EXACT", raising=False)
    monkeypatch.delenv("DCNV4_WINDOW", raising=False)
    if request.param == "window_unit":
        monkeypatch.setenv("DCNV4_WINDOW", "unit")
    elif request.param == "gather":
        monkeypatch.setenv("DCNV4_VARIANT", "gather")
    elif request.param == "window_f16exact":
        monkeypatch.setenv("DCNV4_F16_EXACT", "1")
    return request.param


def _osz(n, K, s, p, d):
    return (n + 2 * p - d * (K - 1) - 1) // s + 1


def _run_case(N, H, W, C, G, K, stride, pad, dil, dtype, offs, v, dev, seed, scale=1.0):
    Ho, Wo = _osz(H, K, stride, pad, dil), _osz(W, K, stride, pad, dil)
    P = K * K - (1 if v.get("remove_center") else 0)
    x, om = make_inputs(N, H, W, C, G, K, Ho, Wo, dtype, offs, ("normal", 0, 1), seed=seed, points=P)
    z = make_center_logit(N, Ho, Wo, G, dtype, seed=seed) if v.get("center") else None
    kw = dict(G=G, K=K, stride=stride, pad=pad, dilation=dil, offset_scale=scale)
    out = dcn.forward(x.to(dev), om.to(dev), softmax=v.get("softmax", False),
                      remove_center=v.get("remove_center", False),
                      center_logit=None if z is None else z.to(dev), **kw)
    torch.cuda.synchronize()
    ref = oracle.dcnv4_forward_variants(x.double().numpy(), om.double().numpy(), softmax=v.get("softmax", False),
                                        remove_center=v.get("remove_center", False),
                                        center_logit=None if z is None else z.double().numpy(), **kw)
    got = out.double().cpu().numpy()
    scale_ = max(np.abs(ref).max(), 1e-30)
    err = np.abs(got - ref).max()
    assert err <= TOL[dtype] * scale_, f"max|err| {err:.3e} > {TOL[dtype]} * {scale_:.3e}"


SHAPES = [
    # N, H, W, C, G, K, stride, pad, dil, offsets
    (2, 13, 11, 64, 4, 3, 1, 1, 1, ("normal", 0, 1.5)),
    (1, 20, 18, 32, 4, 5, 1, 2, 1, ("uniform", -3, 3)),
    (3, 9, 17, 80, 2, 3, 1, 1, 1, ("uniform", -4, 4)),       # Cg 40
    (1, 21, 19, 64, 2, 3, 1, 2, 2, ("uniform", -8, 8)),      # dilation 2
    (1, 16, 16, 128, 8, 3, 2, 1, 1, ("normal", 0, 1)),       # stride 2
    (1, 15, 15, 32, 32, 3, 1, 1, 1, ("normal", 0, 2)),       # Cg 1: element path
]


@pytest.mark.parametrize("vname", list(VARIANTS))
@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("case", SHAPES, ids=lambda c: "x".join(map(str, c[:9])))
def test_variants_match_the_oracle(case, dtype, vname, variant, cuda_device):
    N, H, W, C, G, K, s, p, d, offs = case
    _run_case(N, H, W, C, G, K, s, p, d, dtype, offs, VARIANTS[vname], cuda_device, seed=N * H + C)


@pytest.mark.parametrize("vname", list(VARIANTS))
def test_variants_at_the_stage1_size(vname, variant, cuda_device):
    w = WORKLOADS["stage1_f16"]
    _run_case(w.N, w.H, w.W, w.C, w.G, w.K, w.stride, w.pad, w.dilation, w.dtype, w.offsets, VARIANTS[vname],
              cuda_device, seed=w.seed)


def test_no_flags_is_the_plain_forward_bit_for_bit(cuda_device):
    w = WORKLOADS["stage1_f16"]
    x, om = make_inputs(4, w.H, w.W, w.C, w.G, w.K, w.Hout, w.Wout, w.dtype, w.offsets, w.masks, seed=3)
    x, om = x.to(cuda_device), om.to(cuda_device)
    a = dcn.forward(x, om, **w.kwargs())
    lib = dcn.load_library()
    b = torch.empty_like(a)
    rc = lib.dcnv4_forward_ex(x.data_ptr(), om.data_ptr(), None, b.data_ptr(), 4, w.H, w.W, w.C, w.G, w.K, w.stride,
                              w.pad, w.dilation, w.offset_scale, dcn.DCNV4_F16, 0,
                              torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_saturated_gate_returns_the_centre_feature(dtype, cuda_device):
    # logit +30: s = 1 in fp32, so out = x at the centre position exactly (stride 1, pad 1: x itself)
    N, H, W, C, G, K = 2, 12, 10, 64, 4, 3
    x, om = make_inputs(N, H, W, C, G, K, H, W, dtype, ("normal", 0, 1.5), seed=8)
    z = torch.full((N, H, W, G), 30.0).to(x.dtype)
    out = dcn.forward(x.to(cuda_device), om.to(cuda_device), G=G, K=K, pad=1, center_logit=z.to(cuda_device))
    torch.cuda.synchronize()
    assert torch.equal(out.cpu(), x)
