"""The forward's planner on the host (dcnv4_forward_plan, no GPU): the ring
kernel's shape for the named workloads and a sweep of geometries satisfies the
kernel's own constraints (shared memory, threads, ring depth, window sizes), the
choices that fix each output's summation order (window kind and halo) do not
depend on the batch size, and the overrides and argument checks behave."""
import ctypes

import pytest
import torch

import deformable_convolution_sparse_b200 as dcn
from deformable_convolution_sparse_b200 import binding as B
from deformable_convolution_sparse_b200.workloads import WORKLOADS

DT = {"f32": dcn.DCNV4_F32, "f16": dcn.DCNV4_F16, "bf16": dcn.DCNV4_BF16}
E = {"f32": 4, "f16": 2, "bf16": 2}
SMEM_LIMIT = 226 * 1024


def _osz(n, K, s, p, d):
    return (n + 2 * p - d * (K - 1) - 1) // s + 1


def _plan(N, H, W, C, G, K, s=1, p=0, d=1, dtype="f32", flags=0, nsm=148):
    return dcn.forward_plan(N, H, W, C, G, K, s, p, d, DT[dtype], flags, nsm)


def _check_ring_plan(pl, H, W, C, G, K, s, p, d, dtype):
    Cg = C // G
    Ho, Wo = _osz(H, K, s, p, d), _osz(W, K, s, p, d)
    assert pl["kernel"] == "ring"
    gs = pl["groups_per_strip"]
    assert G % gs == 0
    assert pl["pixel_bytes"] == gs * Cg * E[dtype]
    units = pl["units_per_item"]
    assert units == pl["item_rows"] * pl["band_columns"] * gs
    assert units <= 480 and pl["threads"] == (units + 31) // 32 * 32 + 32
    assert 0 < pl["smem_bytes"] <= SMEM_LIMIT
    assert 2 <= pl["items_in_flight"] <= 4
    if pl["image_windows"]:
        assert pl["unit_window_rows"] == H + 2 and pl["unit_window_cols"] == W + 2
        assert pl["window_pixels"] == W + 2 and pl["band_columns"] == Wo
        rows = pl["unit_window_rows"]
    else:
        R = pl["halo"]
        assert pl["unit_window_rows"] == pl["unit_window_cols"] == (K - 1) * d + 2 * R + 1
        assert pl["window_pixels"] == (pl["band_columns"] - 1) * s + pl["unit_window_cols"]
        rows = (pl["item_rows"] - 1) * s + pl["unit_window_rows"]
    assert pl["window_pixels"] <= 256
    assert pl["ring_rows"] >= rows
    row_pitch = (pl["window_pixels"] * pl["pixel_bytes"] + 127) // 128 * 128
    assert (pl["ring_rows"] + 1) * row_pitch <= pl["smem_bytes"]


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_named_workloads_plan_within_the_kernels_limits(name):
    w = WORKLOADS[name]
    pl = _plan(w.N, w.H, w.W, w.C, w.G, w.K, w.stride, w.pad, w.dilation, w.dtype)
    _check_ring_plan(pl, w.H, w.W, w.C, w.G, w.K, w.stride, w.pad, w.dilation, w.dtype)
    # small images take image windows, the others unit windows with a halo near 4 * dilation + 1
    small = name in ("tiny_f32", "stage3_f16")
    assert pl["image_windows"] == (1 if small else 0)
    if not small:
        assert abs(pl["halo"] - (4 * w.dilation + 1)) <= 1


SHAPES = [
    # H, W, C, G, K, stride, pad, dilation, dtype
    (56, 56, 64, 4, 3, 1, 1, 1, "f16"), (28, 28, 128, 8, 3, 1, 1, 1, "bf16"), (7, 7, 512, 32, 3, 1, 1, 1, "f16"),
    (33, 31, 48, 3, 3, 1, 1, 1, "f32"), (64, 64, 320, 8, 3, 1, 1, 1, "f16"), (100, 37, 256, 8, 5, 2, 2, 1, "f16"),
    (21, 19, 128, 4, 3, 1, 2, 2, "bf16"), (30, 30, 64, 4, 5, 1, 2, 1, "f32"), (12, 12, 64, 8, 1, 1, 0, 1, "f16"),
    (129, 63, 64, 2, 3, 2, 1, 3, "f16"),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda c: "x".join(map(str, c)))
def test_shape_sweep_plans_within_the_kernels_limits(shape):
    H, W, C, G, K, s, p, d, dt = shape
    pl = _plan(16, H, W, C, G, K, s, p, d, dt)
    _check_ring_plan(pl, H, W, C, G, K, s, p, d, dt)


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_window_kind_and_halo_do_not_depend_on_the_batch(name):
    """The window kind and the halo decide which samples take the shared-memory
    path and so the order of each output's sum: they must be the same for every
    batch size (and SM count), so that an image's result never depends on its batch."""
    w = WORKLOADS[name]
    seen = set()
    for N in (1, 2, 7, 64, 500):
        if N * w.H * w.W * w.C >= 2 ** 31 or N * w.Hout * w.Wout * w.G * 27 >= 2 ** 31:
            continue  # beyond the library's element limit
        for nsm in (148, 132):
            pl = _plan(N, w.H, w.W, w.C, w.G, w.K, w.stride, w.pad, w.dilation, w.dtype, nsm=nsm)
            seen.add((pl["kernel"], pl["image_windows"], pl["halo"]))
    assert len(seen) == 1, seen


def test_shapes_the_ring_kernel_does_not_take():
    assert _plan(2, 9, 9, 9, 3, 3, 1, 1, 1, "f16")["kernel"] == "gather"      # 6-byte groups
    assert _plan(2, 30, 30, 64, 4, 9, 1, 4, 1, "f32")["kernel"] == "gather"   # 81 points per unit
    assert _plan(2, 5, 40, 16, 1, 7, 1, 3, 1, "f32")["kernel"] == "gather"    # 49-point records overflow shared memory
    pl = _plan(2, 30, 30, 64, 4, 9, 1, 4, 1, "f32")
    assert all(v == 0 for k, v in pl.items() if k != "kernel")


def test_overrides(monkeypatch):
    w = WORKLOADS["stage3_f16"]
    args = (w.N, w.H, w.W, w.C, w.G, w.K, w.stride, w.pad, w.dilation, w.dtype)
    assert _plan(*args)["image_windows"] == 1
    monkeypatch.setenv("DCNV4_WINDOW", "unit")
    assert _plan(*args)["image_windows"] == 0
    monkeypatch.delenv("DCNV4_WINDOW")
    monkeypatch.setenv("DCNV4_HALO", "3")
    pl = _plan(*args)
    assert pl["image_windows"] == 0 and pl["halo"] == 3
    monkeypatch.delenv("DCNV4_HALO")
    monkeypatch.setenv("DCNV4_GS", "16")
    assert _plan(*args)["groups_per_strip"] == 16
    monkeypatch.delenv("DCNV4_GS")
    assert _plan(*args)["image_windows"] == 1


def test_stage3_image_windows_take_strips_the_ring_can_prefetch():
    # 14x14 images of 16 groups: strips of 8 groups (64 KB windows) in 4-row items, whose ring holds
    # two whole windows, so a CTA's next strip loads during the current one (measured 17.0-17.2 us
    # against 18.4 for strips of all 16 groups, whose 128 KB windows fit only once)
    w = WORKLOADS["stage3_f16"]
    pl = _plan(w.N, w.H, w.W, w.C, w.G, w.K, w.stride, w.pad, w.dilation, w.dtype)
    assert pl["image_windows"] == 1 and pl["groups_per_strip"] == 8 and pl["item_rows"] == 4
    assert pl["ring_rows"] >= 2 * pl["unit_window_rows"]


def test_centre_scaling_keeps_image_windows_only_with_the_centre_inside():
    # pad 1, K 3: every unit's centre grid position lies inside the image window
    assert _plan(4, 14, 14, 64, 4, 3, 1, 1, 1, "f16", flags=B.FLAG_CENTER_SCALE)["image_windows"] == 1
    # pad 3: the first row's centre sits two rows above the image, outside the one-pixel border
    assert _plan(4, 14, 14, 64, 4, 3, 1, 3, 1, "f16", flags=B.FLAG_CENTER_SCALE)["image_windows"] == 0
    assert _plan(4, 14, 14, 64, 4, 3, 1, 3, 1, "f16")["image_windows"] == 1


def test_argument_checks():
    lib = dcn.load_library()
    buf = (ctypes.c_int * dcn.binding.PLAN_FIELDS.__len__())()
    assert lib.dcnv4_forward_plan(2, 8, 8, 16, 2, 3, 1, 1, 1, 0, 0, 148, None, 15) == B.STATUS["DCNV4_ERR_NULL"]
    assert lib.dcnv4_forward_plan(2, 8, 8, 16, 2, 3, 1, 1, 1, 0, 0, 148, buf, 14) == B.STATUS["DCNV4_ERR_SHAPE"]
    assert lib.dcnv4_forward_plan(2, 8, 8, 16, 2, 3, 1, 1, 1, 0, 0, 0, buf, 15) == B.STATUS["DCNV4_ERR_SHAPE"]
    assert lib.dcnv4_forward_plan(2, 8, 8, 16, 2, 3, 1, 1, 1, 0, 64, 148, buf, 15) == B.STATUS["DCNV4_ERR_FLAGS"]
    assert lib.dcnv4_forward_plan(2, 8, 8, 15, 2, 3, 1, 1, 1, 0, 0, 148, buf, 15) == B.STATUS["DCNV4_ERR_GROUPS"]
    assert lib.dcnv4_forward_plan(2, 8, 8, 16, 2, 3, 1, 1, 1, 9, 0, 148, buf, 15) == B.STATUS["DCNV4_ERR_DTYPE"]
    assert lib.dcnv4_forward_plan(0, 8, 8, 16, 2, 3, 1, 1, 1, 0, 0, 148, buf, 15) == dcn.DCNV4_OK
    with pytest.raises(dcn.DCNv4Error):
        dcn.forward_plan(2, 8, 8, 16, 2, 3, nsm=0)
