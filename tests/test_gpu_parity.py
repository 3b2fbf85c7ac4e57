"""GPU parity: the sm_100a kernels (through the C ABI) against the fp64 oracle.

Bars (from the operator's contract): corner indices and validity bit-exact;
max|err| <= 1e-5 * max|out| for fp32 storage and <= 4e-3 * max|out| for
fp16/bf16 storage (fp32 accumulation), with the oracle run on the same
rounded inputs. The five named workloads run at their full sizes in the
launch configuration the benchmark uses.
"""
import math
import zlib

import numpy as np
import pytest
import torch

import oracle
import deformable_convolution_sparse_b200 as dcn
from deformable_convolution_sparse_b200.workloads import WORKLOADS, make_inputs, workload_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "f16": 4e-3, "bf16": 4e-3}
TD = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(params=["window", "window_unit", "window_f16exact", "gather"])
def variant(request, monkeypatch):
    """Every kernel path: the shared-memory ring kernel (default choice: image
    windows for the small images here, unit windows for the large ones; for
    fp16 storage with fp16-rounded weights), the ring kernel held to unit
    windows (DCNV4_WINDOW=unit), the same kernel with fp32 weights for fp16
    (DCNV4_F16_EXACT=1), and the global-gather kernel (forced with
    DCNV4_VARIANT=gather)."""
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


def _check(got: torch.Tensor, ref: np.ndarray, dtype: str, what=""):
    g = got.double().cpu().numpy()
    assert g.shape == ref.shape
    scale = max(np.abs(ref).max(), 1e-30)
    err = np.abs(g - ref).max() if ref.size else 0.0
    assert err <= TOL[dtype] * scale, f"{what}: max|err| {err:.3e} > {TOL[dtype]} * {scale:.3e}"
    return err / scale


def _run_and_check(x, om, dtype, dev, index=True, **kw):
    out = dcn.forward(x.to(dev), om.to(dev), **kw)
    torch.cuda.synchronize()
    ref = oracle.dcnv4_forward(x.double().numpy(), om.double().numpy(), **kw)
    rel = _check(out, ref, dtype)
    if index:
        N, H, W, C = x.shape
        c_gpu, v_gpu = dcn.sampling_index(om.to(dev), H, W, **kw)
        c_ref, v_ref = oracle.sampling_index(om.double().numpy(), H, W, **kw)
        np.testing.assert_array_equal(v_gpu.cpu().numpy(), v_ref)
        np.testing.assert_array_equal(c_gpu.cpu().numpy(), c_ref)
    return out, rel


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_named_workload_full_size(name, variant, cuda_device):
    w = WORKLOADS[name]
    x, om = workload_inputs(w)
    _run_and_check(x, om, w.dtype, cuda_device, **w.kwargs())


SWEEP = [
    # N, H, W, C, G, K, stride, pad, dil, scale, offsets
    (1, 8, 8, 16, 2, 3, 1, 1, 1, 1.0, ("uniform", -2, 2)),
    (2, 13, 11, 64, 4, 3, 1, 1, 1, 1.0, ("normal", 0, 1.5)),
    (3, 9, 17, 80, 2, 3, 1, 1, 1, 1.0, ("uniform", -4, 4)),      # Cg 40
    (1, 15, 15, 32, 32, 3, 1, 1, 1, 0.5, ("normal", 0, 2)),       # Cg 1
    (2, 10, 7, 24, 12, 3, 2, 1, 1, 1.0, ("normal", 0, 1)),        # Cg 2, stride 2
    (1, 9, 9, 9, 3, 3, 1, 2, 2, 1.0, ("uniform", -3, 3)),         # Cg 3, dilation 2
    (2, 11, 12, 16, 4, 5, 1, 2, 1, 0.75, ("normal", 0, 1)),       # Cg 4, K 5
    (1, 12, 12, 64, 8, 1, 1, 0, 1, 1.0, ("normal", 0, 2)),        # Cg 8, K 1
    (1, 7, 9, 128, 2, 3, 2, 1, 1, 1.0, ("normal", 0, 1)),         # Cg 64
    (1, 6, 6, 32, 2, 3, 1, 1, 1, 1.0, ("uniform", -12, 12)),      # many samples fully outside
    (2, 33, 31, 48, 3, 3, 1, 1, 1, 1.0, ("normal", 0, 1.5)),      # Cg 16, odd sizes, ragged tail
    (1, 5, 40, 16, 1, 7, 1, 3, 1, 1.25, ("normal", 0, 3)),        # K 7, G 1
]


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("case", SWEEP, ids=lambda c: "x".join(map(str, c[:9])))
def test_shape_sweep(case, dtype, variant, cuda_device):
    N, H, W, C, G, K, s, p, d, scale, offd = case
    Hout, Wout = _osz(H, K, s, p, d), _osz(W, K, s, p, d)
    x, om = make_inputs(N, H, W, C, G, K, Hout, Wout, dtype, offd, ("normal", 0, 1), seed=zlib.crc32(repr(case).encode()) & 0xffff)
    _run_and_check(x, om, dtype, cuda_device, G=G, K=K, stride=s, pad=p, dilation=d, offset_scale=scale)


def _offset_view(t: torch.Tensor, elems: int, dev):
    """Copy of t placed `elems` elements into a larger buffer (misaligned data pointer)."""
    buf = torch.zeros(t.numel() + elems + 64, dtype=t.dtype, device=dev)
    v = buf[elems:elems + t.numel()].view(t.shape)
    v.copy_(t.to(dev))
    return v


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("shift_x,shift_om,shift_out", [(0, 1, 0), (0, 3, 0), (1, 0, 0), (0, 0, 1), (1, 5, 3)])
def test_misaligned_pointers(dtype, shift_x, shift_om, shift_out, variant, cuda_device):
    N, H, W, C, G, K = 2, 9, 10, 32, 2, 3
    x, om = make_inputs(N, H, W, C, G, K, 9, 10, dtype, ("normal", 0, 1.5), seed=11)
    xd = _offset_view(x, shift_x, cuda_device)
    omd = _offset_view(om, shift_om, cuda_device)
    out = _offset_view(torch.zeros(N, 9, 10, C, dtype=TD[dtype]), shift_out, cuda_device)
    dcn.forward(xd, omd, G=G, K=K, pad=1, out=out)
    torch.cuda.synchronize()
    ref = oracle.dcnv4_forward(x.double().numpy(), om.double().numpy(), G=G, K=K, pad=1)
    _check(out, ref, dtype)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_guard_bands_untouched(dtype, variant, cuda_device):
    N, H, W, C, G, K = 1, 7, 9, 48, 3, 3
    x, om = make_inputs(N, H, W, C, G, K, 7, 9, dtype, ("uniform", -3, 3), seed=12)
    n_out = N * 7 * 9 * C
    guard = 4096
    buf = torch.full((n_out + 2 * guard,), 7.0, dtype=TD[dtype], device=cuda_device)
    out = buf[guard:guard + n_out].view(N, 7, 9, C)
    dcn.forward(x.to(cuda_device), om.to(cuda_device), G=G, K=K, pad=1, out=out)
    torch.cuda.synchronize()
    assert bool((buf[:guard] == 7.0).all()) and bool((buf[guard + n_out:] == 7.0).all())
    _check(out, oracle.dcnv4_forward(x.double().numpy(), om.double().numpy(), G=G, K=K, pad=1), dtype)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("K,dil", [(1, 1), (3, 1), (3, 2), (5, 1)])
def test_identity_is_bit_exact(dtype, K, dil, variant, cuda_device):
    N, H, W, C, G = 2, 11, 13, 64, 4
    KK = K * K
    x = torch.randn(N, H, W, C).to(TD[dtype])
    om = torch.zeros(N, H, W, G, 3 * KK)
    om[..., 2 * KK + (KK - 1) // 2] = 1.0
    out = dcn.forward(x.to(cuda_device), om.to(TD[dtype]).to(cuda_device), G=G, K=K, pad=dil * (K - 1) // 2,
                      dilation=dil)
    torch.cuda.synchronize()
    assert torch.equal(out.cpu(), x)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_mask_and_input_rescaling_is_bit_exact(dtype, cuda_device):
    x, om = make_inputs(2, 16, 16, 64, 4, 3, 16, 16, dtype, ("normal", 0, 1.5), seed=13)
    # keep every x and mask value far from the fp16 subnormal range so that
    # dividing by 4 stays exact
    x = torch.where(x.abs() < 1e-2, torch.full_like(x, 0.25), x)
    m = om[..., 18:]
    om[..., 18:] = torch.where(m.abs() < 1e-2, torch.full_like(m, -0.5), m)
    kw = dict(G=4, K=3, pad=1)
    base = dcn.forward(x.to(cuda_device), om.to(cuda_device), **kw)
    for a in (2.0, 4.0):
        om2 = om.clone()
        om2[..., 18:] *= a
        out = dcn.forward((x / a).to(cuda_device), om2.to(cuda_device), **kw)
        assert torch.equal(out, base)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_far_and_non_finite_offsets_give_exact_zero(dtype, variant, cuda_device):
    N, H, W, C, G, K = 1, 6, 7, 32, 2, 3
    KK = K * K
    x = torch.randn(N, H, W, C).to(TD[dtype])
    vals = [1e4, -1e4, float("inf"), float("-inf"), float("nan"), 3e38 if dtype != "f16" else 6e4]
    for v in vals:
        om = torch.randn(N, H, W, G, 3 * KK)
        om[..., :KK] = v
        out = dcn.forward(x.to(cuda_device), om.to(TD[dtype]).to(cuda_device), G=G, K=K, pad=1)
        assert bool((out == 0).all()), v


def test_nan_in_x_matches_oracle_pattern(variant, cuda_device):
    N, H, W, C, G, K = 1, 6, 6, 16, 1, 1
    x = torch.ones(N, H, W, C)
    x[0, 2, 3, :] = float("nan")
    om = torch.zeros(N, H, W, G, 3)
    om[..., 2] = 1.0
    out = dcn.forward(x.to(cuda_device), om.to(cuda_device), G=G, K=K).cpu().numpy()
    ref = oracle.dcnv4_forward(x.double().numpy(), om.double().numpy(), G=G, K=K)
    np.testing.assert_array_equal(np.isnan(out), np.isnan(ref))
    np.testing.assert_array_equal(np.nan_to_num(out), np.nan_to_num(ref))


def test_empty_batch(cuda_device):
    x = torch.zeros(0, 8, 8, 16, device=cuda_device)
    om = torch.zeros(0, 8, 8, 2, 27, device=cuda_device)
    out = dcn.forward(x, om, G=2, K=3, pad=1)
    assert out.shape == (0, 8, 8, 16)


def test_tiny_images_and_single_pixel(cuda_device):
    for (H, W, K, pad) in [(1, 1, 1, 0), (1, 1, 3, 1), (2, 1, 3, 1), (1, 5, 3, 1)]:
        Hout, Wout = _osz(H, K, 1, pad, 1), _osz(W, K, 1, pad, 1)
        x, om = make_inputs(2, H, W, 16, 2, K, Hout, Wout, "f32", ("uniform", -1.5, 1.5), seed=H * 10 + W)
        _run_and_check(x, om, "f32", cuda_device, G=2, K=K, pad=pad)


def test_offsets_just_below_integers_keep_bit_exact_indices(variant, cuda_device):
    """Offsets of -2^-k and n - 2^-k: floor must not round p0 + d to the integer."""
    N, H, W, C, G, K = 1, 300, 300, 16, 1, 3
    KK = K * K
    om = torch.zeros(N, H, W, G, 3 * KK)
    tiny = torch.tensor([-2.0 ** -k for k in range(1, 25)] + [1 - 2.0 ** -k for k in range(1, 24)] +
                        [-(1 - 2.0 ** -k) for k in range(1, 24)])
    flat = om.view(-1, 3 * KK)
    flat[:, :2 * KK] = tiny[torch.arange(flat.shape[0] * 2 * KK) % tiny.numel()].view(-1, 2 * KK)
    flat[:, 2 * KK:] = 1.0
    x = torch.randn(N, H, W, C)
    _run_and_check(x, om, "f32", cuda_device, G=G, K=K, pad=1)


def test_stream_argument_is_honoured(cuda_device):
    w = WORKLOADS["stage3_f16"]
    x, om = workload_inputs(w)
    xd, omd = x.to(cuda_device), om.to(cuda_device)
    ref = dcn.forward(xd, omd, **w.kwargs())
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        out = dcn.forward(xd, omd, **w.kwargs())
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


@pytest.mark.parametrize("halo", ["1", "2", "6"])
@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_window_halo_sizes(halo, dtype, monkeypatch, cuda_device):
    """Small and large window halos move samples between the shared-memory and
    the global path; the result must not depend on it."""
    monkeypatch.setenv("DCNV4_HALO", halo)
    monkeypatch.delenv("DCNV4_VARIANT", raising=False)
    x, om = make_inputs(2, 21, 19, 128, 4, 3, 21, 19, dtype, ("normal", 0, 2.5), seed=int(halo))
    _run_and_check(x, om, dtype, cuda_device, index=False, G=4, K=3, pad=1)


def test_nan_mask_with_outside_corners(cuda_device):
    """A NaN/Inf mask value reaches the output only through corners inside the image."""
    N, H, W, C, G, K = 1, 8, 8, 64, 4, 3
    x = torch.randn(N, H, W, C)
    om = torch.zeros(N, H, W, G, 27)
    om[..., 18:] = 1.0
    om[0, 0, 0, :, 18] = float("nan")      # k = 0 at (0, 0): corner (-1, -1), all outside
    om[0, 0, 0, :, 0] = -0.5               # ... or half outside
    om[0, 3, 3, :, 22] = float("inf")      # interior sample with an infinite mask
    ref = oracle.dcnv4_forward(x.double().numpy(), om.double().numpy(), G=G, K=K, pad=1)
    for v in ("window", "gather"):
        import os
        os.environ["DCNV4_VARIANT"] = v
        try:
            out = dcn.forward(x.to(cuda_device), om.to(cuda_device), G=G, K=K, pad=1).cpu().double().numpy()
        finally:
            del os.environ["DCNV4_VARIANT"]
        np.testing.assert_array_equal(np.isnan(out), np.isnan(ref))
        np.testing.assert_array_equal(np.isinf(out), np.isinf(ref))
        fin = np.isfinite(ref)
        np.testing.assert_allclose(out[fin], ref[fin], rtol=0, atol=1e-5 * np.abs(ref[fin]).max())


def test_bounded_wait_selftest_sets_status_and_context_survives(cuda_device):
    """The bulk-copy waits give up after a time limit and report through the
    device status word; the self test makes such a wait run out on purpose
    (an mbarrier armed for bytes nobody sends) without faulting anything."""
    st0 = dcn.device_status(clear=True)
    assert not st0 & dcn.binding.DEVSTATUS_COPY_TIMEOUT
    dcn.selftest_wait_timeout(2_000_000)
    torch.cuda.synchronize()
    st = dcn.device_status(clear=True)
    assert st & dcn.binding.DEVSTATUS_SELFTEST_TIMEOUT
    assert not st & dcn.binding.DEVSTATUS_COPY_TIMEOUT
    assert dcn.device_status() == 0
    # the context is still healthy: a forward still matches the oracle
    w = WORKLOADS["tiny_f32"]
    x, om = workload_inputs(w)
    _run_and_check(x, om, "f32", cuda_device, **w.kwargs())


def test_no_copy_timeouts_during_the_parity_runs(cuda_device):
    st = dcn.device_status(clear=True)
    assert not st & dcn.binding.DEVSTATUS_COPY_TIMEOUT


@pytest.mark.parametrize("name", ["stage1_f16", "stage3_f16", "sd_latent_f16"])
def test_fp16_weight_rounding_stays_far_inside_the_tolerance(name, monkeypatch, cuda_device):
    """fp16 storage: the default path rounds each bilinear weight to fp16
    before the exact fp16 x fp16 product; its error against the oracle must
    stay a small fraction of the 4e-3 * max|out| bar, and close to the error of
    the fp32-weight path."""
    w = WORKLOADS[name]
    x, om = workload_inputs(w)
    ref = oracle.dcnv4_forward(x.double().numpy(), om.double().numpy(), **w.kwargs())
    scale = np.abs(ref).max()
    errs = {}
    for exact in ("0", "1"):
        monkeypatch.setenv("DCNV4_F16_EXACT", exact)
        out = dcn.forward(x.to(cuda_device), om.to(cuda_device), **w.kwargs())
        errs[exact] = np.abs(out.double().cpu().numpy() - ref).max() / scale
    assert errs["0"] <= 1e-3, errs        # a quarter of the 4e-3 bar
    assert errs["0"] <= 2.0 * errs["1"] + 2e-4, errs


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_an_image_result_does_not_depend_on_its_batch(dtype, cuda_device):
    """Batch invariance: the kernel choice and tiling depend on the image
    geometry only, so every image gives the same bits alone or in a batch."""
    x, om = make_inputs(12, 40, 44, 64, 4, 3, 40, 44, dtype, ("normal", 0, 2.5), ("normal", 0, 0.5), seed=31)
    full = dcn.forward(x.to(cuda_device), om.to(cuda_device), G=4, K=3, pad=1).cpu()
    for lo, hi in [(0, 1), (3, 8), (11, 12)]:
        part = dcn.forward(x[lo:hi].contiguous().to(cuda_device), om[lo:hi].contiguous().to(cuda_device),
                           G=4, K=3, pad=1).cpu()
        assert torch.equal(part, full[lo:hi]), (lo, hi)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_chained_launches_read_the_previous_output(dtype, monkeypatch, cuda_device):
    """Each forward of a chain reads the previous one's output as its input, with
    no synchronisation between the launches (the ring kernel is launched with
    programmatic stream serialisation and waits for the grid before it): the
    chain must give the bits of the same chain run launch by launch, and of
    the same chain with plain serialisation (DCNV4_PDL=0)."""
    monkeypatch.delenv("DCNV4_VARIANT", raising=False)
    N, H, W, C, G, K = 16, 28, 28, 64, 4, 3
    x, om = make_inputs(N, H, W, C, G, K, H, W, dtype, ("normal", 0, 1.5), ("normal", 0, 0.5), seed=61)
    oms = [om.roll(i, dims=0).to(cuda_device) for i in range(6)]

    def chain(sync):
        cur = x.to(cuda_device)
        for o in oms:
            cur = dcn.forward(cur, o, G=G, K=K, pad=1)
            if sync:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        return cur

    fast = chain(False)
    stepwise = chain(True)
    monkeypatch.setenv("DCNV4_PDL", "0")
    plain = chain(False)
    ity = torch.int32 if fast.element_size() == 4 else torch.int16
    assert torch.equal(fast.view(ity), stepwise.view(ity))
    assert torch.equal(fast.view(ity), plain.view(ity))
