"""GPU parity of the backward with the variant flags (dcnv4_backward_ex:
softmax over the masks, centre point removed, centre feature scaling, all
three) against the oracle's variant backward; bars as the plain backward's
(max|err| <= 1e-5 * max|ref| per gradient block, for every storage dtype)."""
import numpy as np
import pytest
import torch

import oracle
import deformable_convolution_sparse_b200 as dcn
from deformable_convolution_sparse_b200.workloads import WORKLOADS, make_center_logit, make_grad_out, make_inputs

pytestmark = pytest.mark.gpu

TOL = 1e-5
VARIANTS = {
    "softmax": dict(softmax=True),
    "remove_center": dict(remove_center=True),
    "center_scale": dict(center=True),
    "all": dict(softmax=True, remove_center=True, center=True),
}


def _osz(n, K, s, p, d):
    return (n + 2 * p - d * (K - 1) - 1) // s + 1


def _block(got, ref, what):
    scale = max(float(np.abs(ref).max()), 1e-30)
    err = float(np.abs(got - ref).max())
    assert err <= TOL * scale, f"{what}: max|err| {err:.3e} > {TOL} * {scale:.3e}"


def _run(N, H, W, C, G, K, stride, pad, dil, dtype, offs, v, dev, seed):
    Ho, Wo = _osz(H, K, stride, pad, dil), _osz(W, K, stride, pad, dil)
    P = K * K - (1 if v.get("remove_center") else 0)
    x, om = make_inputs(N, H, W, C, G, K, Ho, Wo, dtype, offs, ("normal", 0, 1), seed=seed, points=P)
    go = make_grad_out(N, Ho, Wo, C, dtype, seed=seed)
    z = make_center_logit(N, Ho, Wo, G, dtype, seed=seed) if v.get("center") else None
    kw = dict(G=G, K=K, stride=stride, pad=pad, dilation=dil)
    res = dcn.backward(x.to(dev), om.to(dev), go.to(dev), softmax=v.get("softmax", False),
                       remove_center=v.get("remove_center", False),
                       center_logit=None if z is None else z.to(dev), **kw)
    torch.cuda.synchronize()
    rgx, rgom, rgz = oracle.dcnv4_backward_variants(x.double().numpy(), om.double().numpy(), go.double().numpy(),
                                                    softmax=v.get("softmax", False),
                                                    remove_center=v.get("remove_center", False),
                                                    center_logit=None if z is None else z.double().numpy(), **kw)
    _block(res[0].cpu().numpy().astype(np.float64), rgx, "grad_x")
    gom = res[1].cpu().numpy().astype(np.float64)
    for i, name in enumerate(("grad_offset_x", "grad_offset_y", "grad_mask")):
        _block(gom[..., i * P:(i + 1) * P], rgom[..., i * P:(i + 1) * P], name)
    if z is not None:
        assert len(res) == 3
        _block(res[2].cpu().numpy().astype(np.float64), rgz, "grad_center_logit")
    else:
        assert len(res) == 2


SHAPES = [
    # N, H, W, C, G, K, stride, pad, dil, offsets
    (2, 13, 11, 64, 4, 3, 1, 1, 1, ("normal", 0, 1.5)),
    (1, 20, 18, 32, 4, 5, 1, 2, 1, ("uniform", -3, 3)),
    (3, 9, 17, 80, 2, 3, 1, 1, 1, ("uniform", -4, 4)),       # Cg 40
    (1, 16, 16, 128, 8, 3, 2, 1, 1, ("normal", 0, 1)),       # stride 2
    (1, 15, 15, 32, 32, 3, 1, 1, 1, ("normal", 0, 2)),       # Cg 1: element path
    (1, 9, 9, 1024, 2, 3, 1, 1, 1, ("normal", 0, 1)),        # more chunks than lanes
]


@pytest.mark.parametrize("vname", list(VARIANTS))
@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("case", SHAPES, ids=lambda c: "x".join(map(str, c[:9])))
def test_variant_backward_matches_the_oracle(case, dtype, vname, cuda_device):
    N, H, W, C, G, K, s, p, d, offs = case
    _run(N, H, W, C, G, K, s, p, d, dtype, offs, VARIANTS[vname], cuda_device, seed=N * H + C)


@pytest.mark.parametrize("vname", list(VARIANTS))
def test_variant_backward_at_the_stage1_size(vname, cuda_device):
    w = WORKLOADS["stage1_f16"]
    _run(w.N, w.H, w.W, w.C, w.G, w.K, w.stride, w.pad, w.dilation, w.dtype, w.offsets, VARIANTS[vname],
         cuda_device, seed=w.seed)


def test_no_flags_through_the_ex_entry_is_the_plain_backward(cuda_device):
    w = WORKLOADS["tiny_f32"]
    x, om = (t.to(cuda_device) for t in make_inputs(2, 8, 8, 16, 2, 3, 8, 8, "f32", seed=3))
    go = make_grad_out(2, 8, 8, 16, "f32", seed=3).to(cuda_device)
    a = dcn.backward(x, om, go, G=2, K=3, pad=1)
    lib = dcn.load_library()
    gx, gom = torch.empty_like(a[0]), torch.empty_like(a[1])
    rc = lib.dcnv4_backward_ex(x.data_ptr(), om.data_ptr(), None, go.data_ptr(), gx.data_ptr(), gom.data_ptr(), None,
                               2, 8, 8, 16, 2, 3, 1, 1, 1, 1.0, dcn.DCNV4_F32, 0,
                               torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert torch.equal(a[1], gom)
    assert (a[0] - gx).abs().max().item() <= 1e-6 * a[0].abs().max().item()
