"""GPU: the corner indices and validity that the forward kernels actually use,
bit for bit against the fp64 oracle.

``dcnv4_forward_trace`` runs the forward through the same plan and kernel code
as ``dcnv4_forward`` (a separate build of the ring kernel with trace stores
compiled in) and records, per sampling point, the top-left corner, the
validity bits and the path of the gather: the ring kernel's shared-memory
window (corner read back from the window address arithmetic, path 0), its
global-memory pass (1), the global-gather kernel (2), or none: a sample
outside an image window, which has no corner inside the image (3). The corners and validity must
equal the oracle's (the sample sits at the regular grid position plus the
learned offset: "不只是卷积的平替", jsqmd.com, section 1), and the output must be
the plain forward's bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import deformable_convolution_sparse_b200 as dcn
from deformable_convolution_sparse_b200.workloads import WORKLOADS, make_inputs, workload_inputs

pytestmark = pytest.mark.gpu


def _trace_and_check(x, om, dev, **kw):
    xd, omd = x.to(dev), om.to(dev)
    out, trace = dcn.forward_trace(xd, omd, **kw)
    plain = dcn.forward(xd, omd, **kw)
    torch.cuda.synchronize()
    ity = torch.int32 if out.element_size() == 4 else torch.int16
    assert torch.equal(out.view(ity), plain.view(ity)), "the traced forward must write the plain forward's bits"
    N, H, W, C = x.shape
    c_ref, v_ref = oracle.sampling_index(om.double().numpy(), H, W, **kw)
    t = trace.cpu().numpy()
    np.testing.assert_array_equal(t[..., 2].astype(np.uint8), v_ref)
    np.testing.assert_array_equal(t[..., :2], c_ref)
    return t[..., 3]


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_named_workload_corners_are_bit_exact(name, cuda_device):
    w = WORKLOADS[name]
    x, om = workload_inputs(w)
    path = _trace_and_check(x, om, cuda_device, **w.kwargs())
    # the ring kernel takes every one: the shared-memory window serves the samples
    # (or, for an image window, skips those with no corner inside the image)
    assert (path != 2).all()
    assert np.isin(path, (0, 3)).mean() > 0.9, np.bincount(path.ravel())
    # the paths agree with the plan the library reports for this geometry
    dt = {"f32": dcn.DCNV4_F32, "f16": dcn.DCNV4_F16, "bf16": dcn.DCNV4_BF16}[w.dtype]
    plan = dcn.forward_plan(w.N, w.H, w.W, w.C, w.G, w.K, w.stride, w.pad, w.dilation, dt)
    assert plan["kernel"] == "ring"
    if not plan["image_windows"]:
        assert not (path == 3).any()


def test_offsets_just_below_integers(cuda_device):
    """Offsets of -2^-k, 1 - 2^-k and -(1 - 2^-k): floor(p0 + d) must not round to the integer."""
    N, H, W, C, G, K = 1, 300, 300, 16, 1, 3
    KK = K * K
    om = torch.zeros(N, H, W, G, 3 * KK)
    tiny = torch.tensor([-2.0 ** -k for k in range(1, 25)] + [1 - 2.0 ** -k for k in range(1, 24)] +
                        [-(1 - 2.0 ** -k) for k in range(1, 24)])
    flat = om.view(-1, 3 * KK)
    flat[:, :2 * KK] = tiny[torch.arange(flat.shape[0] * 2 * KK) % tiny.numel()].view(-1, 2 * KK)
    flat[:, 2 * KK:] = 1.0
    x = torch.randn(N, H, W, C)
    path = _trace_and_check(x, om, cuda_device, G=G, K=K, pad=1)
    assert (path == 0).all()


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("window", ["unit", "image"])
def test_window_kinds_route_far_samples(window, dtype, monkeypatch, cuda_device):
    """Offsets of several image widths: a unit window sends its far samples to
    the global-memory pass, an image window skips them (no corner of theirs is
    inside the image); near samples take the shared-memory window either way.
    Corners and validity must be the oracle's on every path."""
    monkeypatch.setenv("DCNV4_WINDOW", window)
    x, om = make_inputs(3, 17, 15, 64, 4, 3, 17, 15, dtype, ("normal", 0, 9), seed=31)
    path = _trace_and_check(x, om, cuda_device, G=4, K=3, pad=1)
    assert (path == 0).any()
    if window == "unit":
        assert set(np.unique(path)) == {0, 1}
    else:
        assert set(np.unique(path)) == {0, 3}


def test_image_window_non_finite_masks_take_the_global_pass(monkeypatch, cuda_device):
    """An image window sends a sample with a non-finite mask and a corner
    inside the image to the global pass, where only valid corners add (NaN or
    Inf reaches those outputs alone)."""
    monkeypatch.setenv("DCNV4_WINDOW", "image")
    N, H, W, C, G, K = 2, 10, 12, 32, 2, 3
    x, om = make_inputs(N, H, W, C, G, K, H, W, "f32", ("normal", 0, 3), seed=41)
    flat = om.view(-1, 27)
    vals = torch.tensor([float("nan"), float("inf"), -float("inf")])
    flat[::5, 18 + 4] = vals[torch.arange(flat[::5].shape[0]) % 3]
    path = _trace_and_check(x, om, cuda_device, G=G, K=K, pad=1)
    assert (path == 1).any() and set(np.unique(path)) <= {0, 1, 3}
    out = dcn.forward(x.to(cuda_device), om.to(cuda_device), G=G, K=K, pad=1).cpu().double().numpy()
    ref = oracle.dcnv4_forward(x.double().numpy(), om.double().numpy(), G=G, K=K, pad=1)
    fin = np.isfinite(ref)
    np.testing.assert_array_equal(np.isfinite(out), fin)
    np.testing.assert_array_equal(np.isnan(out), np.isnan(ref))
    assert np.abs(out[fin] - ref[fin]).max() <= 1e-5 * np.abs(ref[fin]).max()


@pytest.mark.parametrize("halo", ["1", "2", "6"])
@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_halo_sizes_split_points_between_paths(halo, dtype, monkeypatch, cuda_device):
    """Small halos send many samples to the global-memory pass; every corner must
    still be the oracle's, on both paths."""
    monkeypatch.setenv("DCNV4_HALO", halo)
    x, om = make_inputs(2, 21, 19, 128, 4, 3, 21, 19, dtype, ("normal", 0, 2.5), seed=int(halo))
    path = _trace_and_check(x, om, cuda_device, G=4, K=3, pad=1)
    assert (path == 0).any() and (path == 1).any()


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_non_finite_and_far_offsets(dtype, cuda_device):
    N, H, W, C, G, K = 1, 12, 13, 64, 4, 3
    x, om = make_inputs(N, H, W, C, G, K, H, W, dtype, ("normal", 0, 2), seed=21)
    om = om.float()
    flat = om.view(-1, 27)
    vals = torch.tensor([float("nan"), float("inf"), -float("inf"), 1e4, -1e4, 12.5, -13.25])
    flat[::3, 0] = vals[torch.arange(flat[::3].shape[0]) % vals.numel()]
    flat[1::3, 9 + 4] = vals[torch.arange(flat[1::3].shape[0]) % vals.numel()]
    om = om.to(x.dtype)
    _trace_and_check(x, om, cuda_device, G=G, K=K, pad=1)


def test_strided_dilated_and_other_kernel_sizes(cuda_device):
    for (N, H, W, C, G, K, s, p, d, dt) in [(2, 23, 29, 64, 4, 3, 2, 1, 1, "f16"), (1, 30, 30, 64, 2, 5, 1, 2, 1, "f32"),
                                           (2, 40, 36, 128, 8, 3, 1, 2, 2, "bf16"), (1, 17, 19, 80, 2, 3, 1, 1, 1, "f16")]:
        Ho, Wo = (H + 2 * p - d * (K - 1) - 1) // s + 1, (W + 2 * p - d * (K - 1) - 1) // s + 1
        x, om = make_inputs(N, H, W, C, G, K, Ho, Wo, dt, ("normal", 0, 3), seed=H + K)
        _trace_and_check(x, om, cuda_device, G=G, K=K, stride=s, pad=p, dilation=d)


def test_gather_kernel_shapes_are_traced_too(cuda_device):
    # Cg = 3 (6 bytes per group in fp16): the ring kernel does not take it
    x, om = make_inputs(1, 9, 9, 9, 3, 3, 9, 9, "f16", ("uniform", -3, 3), seed=9)
    path = _trace_and_check(x, om, cuda_device, G=3, K=3, pad=1)
    assert (path == 2).all()
