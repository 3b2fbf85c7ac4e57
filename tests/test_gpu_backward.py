"""GPU parity of the backward (dcnv4_backward through the C ABI) against the
fp64 oracle's backward, on the same rounded inputs.

Bar: both gradients are fp32 sums of fp32 products of the stored values, so
for every storage dtype max|err| <= 1e-5 * max|ref|, taken separately for
grad_x and for each of the three blocks of the gradient record (x-offsets,
y-offsets, masks), whose scales differ. The named workloads run at full size.
"""
import numpy as np
import pytest
import torch

import oracle
import deformable_convolution_sparse_b200 as dcn
from deformable_convolution_sparse_b200.workloads import (WORKLOADS, make_grad_out, make_inputs, workload_grad_out,
                                                          workload_inputs)

pytestmark = pytest.mark.gpu

TOL = 1e-5


def _osz(n, K, s, p, d):
    return (n + 2 * p - d * (K - 1) - 1) // s + 1


def _check_block(got: np.ndarray, ref: np.ndarray, what: str):
    assert got.shape == ref.shape, what
    if ref.size == 0:
        return 0.0
    scale = max(float(np.abs(ref).max()), 1e-30)
    err = float(np.abs(got - ref).max())
    assert err <= TOL * scale, f"{what}: max|err| {err:.3e} > {TOL} * {scale:.3e}"
    return err / scale


def _check_grads(gx, gom, x, om, go, K, **kw):
    rgx, rgom = oracle.dcnv4_backward(x.double().numpy(), om.double().numpy(), go.double().numpy(), K=K, **kw)
    gx = gx.cpu().numpy().astype(np.float64)
    gom = gom.cpu().numpy().astype(np.float64)
    KK = K * K
    rel = [_check_block(gx, rgx, "grad_x")]
    for i, name in enumerate(("grad_offset_x", "grad_offset_y", "grad_mask")):
        rel.append(_check_block(gom[..., i * KK:(i + 1) * KK], rgom[..., i * KK:(i + 1) * KK], name))
    return rel


def _run(x, om, go, dev, K, **kw):
    gx, gom = dcn.backward(x.to(dev), om.to(dev), go.to(dev), K=K, **kw)
    torch.cuda.synchronize()
    return gx, gom


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_named_workload_full_size(name, cuda_device):
    w = WORKLOADS[name]
    x, om = workload_inputs(w)
    go = workload_grad_out(w)
    kw = w.kwargs()
    gx, gom = _run(x, om, go, cuda_device, **kw)
    _check_grads(gx, gom, x, om, go, **kw)


SWEEP = [
    # N, H, W, C, G, K, stride, pad, dil, scale, offsets
    (1, 8, 8, 16, 2, 3, 1, 1, 1, 1.0, ("uniform", -2, 2)),
    (2, 13, 11, 64, 4, 3, 1, 1, 1, 1.0, ("normal", 0, 1.5)),
    (3, 9, 17, 80, 2, 3, 1, 1, 1, 1.0, ("uniform", -4, 4)),      # Cg 40
    (1, 15, 15, 32, 32, 3, 1, 1, 1, 0.5, ("normal", 0, 2)),       # Cg 1: element path
    (2, 12, 10, 24, 2, 3, 1, 1, 1, 1.0, ("normal", 0, 1)),        # Cg 12: element path for fp16
    (1, 16, 16, 128, 1, 3, 2, 1, 1, 1.0, ("normal", 0, 1)),       # Cg 128, stride 2
    (1, 20, 18, 32, 4, 5, 1, 2, 1, 2.0, ("uniform", -3, 3)),      # K 5
    (2, 10, 10, 64, 8, 1, 1, 0, 1, 1.0, ("normal", 0, 0.7)),      # K 1
    (1, 21, 19, 64, 2, 3, 1, 2, 2, 1.0, ("uniform", -8, 8)),      # dilation 2
    (5, 7, 9, 48, 3, 3, 1, 1, 1, 1.0, ("normal", 0, 3)),          # ragged unit count
    (1, 9, 9, 1024, 2, 3, 1, 1, 1, 1.0, ("normal", 0, 1)),        # Cg 512: more chunks than lanes
]


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("case", SWEEP, ids=lambda c: "x".join(map(str, c[:9])))
def test_shape_sweep(case, dtype, cuda_device):
    N, H, W, C, G, K, s, p, d, sc, offs = case
    Ho, Wo = _osz(H, K, s, p, d), _osz(W, K, s, p, d)
    x, om = make_inputs(N, H, W, C, G, K, Ho, Wo, dtype, offs, ("normal", 0, 1), seed=N * H + C)
    go = make_grad_out(N, Ho, Wo, C, dtype, seed=C + K)
    kw = dict(G=G, stride=s, pad=p, dilation=d, offset_scale=sc)
    gx, gom = _run(x, om, go, cuda_device, K, **kw)
    _check_grads(gx, gom, x, om, go, K, **kw)


def _offset_view(t: torch.Tensor, elems: int, dev):
    flat = torch.empty(t.numel() + elems, dtype=t.dtype, device=dev)
    v = flat[elems:].view(t.shape)
    v.copy_(t.to(dev))
    return v


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("shift_x,shift_om,shift_go,shift_gx", [(1, 0, 0, 0), (0, 3, 0, 0), (0, 0, 1, 0),
                                                                 (0, 0, 0, 1), (1, 5, 3, 2)])
def test_misaligned_pointers(dtype, shift_x, shift_om, shift_go, shift_gx, cuda_device):
    N, H, W, C, G, K = 2, 11, 13, 64, 4, 3
    x, om = make_inputs(N, H, W, C, G, K, H, W, dtype, ("normal", 0, 1.5), ("normal", 0, 1), seed=9)
    go = make_grad_out(N, H, W, C, dtype, seed=9)
    xd, omd, god = (_offset_view(t, sft, cuda_device) for t, sft in ((x, shift_x), (om, shift_om), (go, shift_go)))
    gx = _offset_view(torch.zeros(N, H, W, C), shift_gx, cuda_device)
    gom = _offset_view(torch.zeros(N, H, W, G, 3 * K * K), 1, cuda_device)
    dcn.backward(xd, omd, god, G=G, K=K, pad=1, grad_x=gx, grad_offset_mask=gom)
    torch.cuda.synchronize()
    _check_grads(gx, gom, x, om, go, K, G=G, pad=1)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_far_and_non_finite_offsets_give_exact_zeros(dtype, cuda_device):
    N, H, W, C, G, K = 2, 9, 9, 32, 2, 3
    KK = K * K
    x, om = make_inputs(N, H, W, C, G, K, H, W, dtype, seed=4)
    go = make_grad_out(N, H, W, C, dtype, seed=4)
    bad = om.clone()
    vals = torch.tensor([float(H + W + 5), -1e4, float("inf"), float("nan")]).to(bad.dtype)
    bad[..., :KK] = vals[torch.arange(bad[..., :KK].numel()) % 4].view(bad[..., :KK].shape)
    gx, gom = _run(x, bad, go, cuda_device, K, G=G, pad=1)
    assert not gx.any() and not gom.any()


def test_grad_out_may_share_memory_with_x(cuda_device):
    # stride 1, pad 1, K 3: grad_out has x's shape; both are read only
    N, H, W, C, G, K = 2, 10, 12, 32, 4, 3
    x, om = make_inputs(N, H, W, C, G, K, H, W, "f32", ("normal", 0, 1), seed=13)
    xd = x.to(cuda_device)
    gx, gom = dcn.backward(xd, om.to(cuda_device), xd, G=G, K=K, pad=1)
    torch.cuda.synchronize()
    _check_grads(gx, gom, x, om, x, K, G=G, pad=1)


def test_gradient_record_is_deterministic_and_grad_x_reproducible(cuda_device):
    w = WORKLOADS["stage1_f16"]
    x, om = (t.to(cuda_device) for t in workload_inputs(w))
    go = workload_grad_out(w).to(cuda_device)
    a = dcn.backward(x, om, go, **w.kwargs())
    b = dcn.backward(x, om, go, **w.kwargs())
    torch.cuda.synchronize()
    assert torch.equal(a[1], b[1])
    scale = a[0].abs().max().item()
    assert (a[0] - b[0]).abs().max().item() <= 1e-6 * scale


def test_outputs_are_overwritten_and_guard_bands_untouched(cuda_device):
    N, H, W, C, G, K = 1, 12, 12, 64, 4, 3
    x, om = make_inputs(N, H, W, C, G, K, H, W, "f16", ("normal", 0, 1.5), seed=21)
    go = make_grad_out(N, H, W, C, "f16", seed=21)
    nx, nom, guard = N * H * W * C, N * H * W * G * 3 * K * K, 64
    gxb = torch.full((nx + 2 * guard,), 7.0, device=cuda_device)
    gomb = torch.full((nom + 2 * guard,), 7.0, device=cuda_device)
    gx, gom = gxb[guard:guard + nx].view(N, H, W, C), gomb[guard:guard + nom].view(N, H, W, G, 3 * K * K)
    dcn.backward(x.to(cuda_device), om.to(cuda_device), go.to(cuda_device), G=G, K=K, pad=1, grad_x=gx,
                 grad_offset_mask=gom)
    torch.cuda.synchronize()
    for buf in (gxb, gomb):
        assert torch.all(buf[:guard] == 7.0) and torch.all(buf[-guard:] == 7.0)
    _check_grads(gx, gom, x, om, go, K, G=G, pad=1)


def test_adjoint_of_the_gpu_forward(cuda_device):
    # <forward(x), g> = <x, grad_x>, both sides from the GPU paths, fp32 storage, full stage-1 size
    w = WORKLOADS["stage1_f32"]
    x, om = (t.to(cuda_device) for t in workload_inputs(w))
    go = workload_grad_out(w).to(cuda_device)
    out = dcn.forward(x, om, **w.kwargs())
    gx, _ = dcn.backward(x, om, go, **w.kwargs())
    lhs = (out.double() * go.double()).sum().item()
    rhs = (x.double() * gx.double()).sum().item()
    assert abs(lhs - rhs) <= 1e-5 * (out.double().abs() * go.double().abs()).sum().item()


def test_empty_batch(cuda_device):
    x = torch.zeros(0, 8, 8, 16, device=cuda_device)
    om = torch.zeros(0, 8, 8, 2, 27, device=cuda_device)
    gx, gom = dcn.backward(x, om, torch.zeros(0, 8, 8, 16, device=cuda_device), G=2, K=3, pad=1)
    assert gx.shape == (0, 8, 8, 16) and gom.shape == (0, 8, 8, 2, 27)


def test_stream_argument_is_honoured(cuda_device):
    w = WORKLOADS["tiny_f32"]
    x, om = (t.to(cuda_device) for t in workload_inputs(w))
    go = workload_grad_out(w).to(cuda_device)
    s = torch.cuda.Stream(device=cuda_device)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        gx, gom = dcn.backward(x, om, go, stream=s, **w.kwargs())
    s.synchronize()
    _check_grads(gx, gom, x.cpu(), om.cpu(), go.cpu(), **w.kwargs())
