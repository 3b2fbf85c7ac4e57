"""Pins for the fp64 oracle: checks that do not reuse the oracle's code.

Each test fixes the oracle against something other than itself: values worked
out by hand (tests/golden/hand_cases.json), closed forms (identity, shifts,
half-integer offsets, partition of unity), library routines (torch
``grid_sample`` in fp64 for fractional offsets), brute-force integer gathers
written with numpy indexing, and structural invariants (linearity,
out-of-bounds zeros, group equivalence, translation equivariance).

Definition: "不只是卷积的平替：我把DCNv4塞进Stable Diffusion的U-Net里" (jsqmd.com),
section 1 (no softmax; the simplified forward listing), and the usage guide
"掌握DCNv4技术" (pwwt.cn), tuning section (offset_scale).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from deformable_convolution_sparse_b200.workloads import WORKLOADS, workload_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")


def _om(off_x, off_y, mask):
    """Pack [..., KK] planes into the per-group record [dx | dy | m]."""
    return np.concatenate([off_x, off_y, mask], axis=-1)


def _osz(n, K, s, p, d):
    return (n + 2 * p - d * (K - 1) - 1) // s + 1


# ----------------------------------------------------------------- golden ---

def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


def _golden_inputs(case):
    sh = case["shape"]
    N, H, W, C = sh["N"], sh["H"], sh["W"], sh["C"]
    G, K = sh["G"], sh["K"]
    Hout = _osz(H, K, sh["stride"], sh["pad"], sh["dilation"])
    Wout = _osz(W, K, sh["stride"], sh["pad"], sh["dilation"])
    if "x" in case:
        x = np.array(case["x"], dtype=np.float64)
    elif case["name"] == "k3_grid_order":
        x = np.zeros((N, H, W, C))
        for y in range(H):
            for xx in range(W):
                x[0, y, xx, 0] = 3 * y + xx + 1
    else:
        x = np.zeros((N, H, W, C))
        for y in range(H):
            for xx in range(W):
                x[0, y, xx, 0] = 4 * y + xx
                x[0, y, xx, 1] = 10 * y + xx
    if "offset_mask" in case:
        om = np.array(case["offset_mask"], dtype=np.float64)
    else:
        KK = K * K
        om = np.zeros((N, Hout, Wout, G, 3 * KK))
        om[..., 2 * KK:] = np.arange(1, KK + 1, dtype=np.float64)
    return x, om


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_golden_hand_cases(case):
    sh = case["shape"]
    x, om = _golden_inputs(case)
    kw = dict(G=sh["G"], K=sh["K"], stride=sh["stride"], pad=sh["pad"],
              dilation=sh["dilation"], offset_scale=sh["offset_scale"])
    out = oracle.dcnv4_forward(x, om, **kw)
    np.testing.assert_array_equal(out, np.array(case["out"], dtype=np.float64))
    if "corner" in case:
        corner, valid = oracle.sampling_index(om, x.shape[1], x.shape[2], **kw)
        np.testing.assert_array_equal(corner, np.array(case["corner"], dtype=np.int32))
        np.testing.assert_array_equal(valid, np.array(case["valid"], dtype=np.uint8))


# ------------------------------------------------------------ closed forms ---

@pytest.mark.parametrize("K,dil", [(1, 1), (3, 1), (3, 2), (5, 1), (7, 3)])
def test_identity_with_centre_one_hot(K, dil):
    rng = np.random.default_rng(K * 10 + dil)
    N, H, W, C, G = 2, 9, 11, 6, 3
    pad = dil * (K - 1) // 2
    KK = K * K
    x = rng.standard_normal((N, H, W, C))
    m = np.zeros((N, H, W, G, KK))
    m[..., (KK - 1) // 2] = 1.0
    z = np.zeros((N, H, W, G, KK))
    out = oracle.dcnv4_forward(x, _om(z, z, m), G=G, K=K, pad=pad, dilation=dil)
    np.testing.assert_array_equal(out, x)


def test_grid_point_and_offset_axis_order():
    rng = np.random.default_rng(1)
    N, H, W, C, G, K = 1, 6, 7, 4, 2, 3
    KK = K * K
    x = rng.integers(-8, 8, size=(N, H, W, C)).astype(np.float64)
    z = np.zeros((N, H, W, G, KK))
    xp = np.pad(x, ((0, 0), (1, 1), (1, 1), (0, 0)))
    # one-hot at k = 1 (ky = 0, kx = 1): out[ho, wo] = x[ho - 1, wo]
    m = np.zeros_like(z)
    m[..., 1] = 1.0
    out = oracle.dcnv4_forward(x, _om(z, z, m), G=G, K=K, pad=1)
    np.testing.assert_array_equal(out, xp[:, 0:H, 1:W + 1])
    # one-hot at k = 3 (ky = 1, kx = 0): out[ho, wo] = x[ho, wo - 1]
    m = np.zeros_like(z)
    m[..., 3] = 1.0
    out = oracle.dcnv4_forward(x, _om(z, z, m), G=G, K=K, pad=1)
    np.testing.assert_array_equal(out, xp[:, 1:H + 1, 0:W])
    # centre point with the first offset block = +1: moves along the width
    m = np.zeros_like(z)
    m[..., 4] = 1.0
    dx = np.zeros_like(z)
    dx[..., 4] = 1.0
    out = oracle.dcnv4_forward(x, _om(dx, z, m), G=G, K=K, pad=1)
    np.testing.assert_array_equal(out, xp[:, 1:H + 1, 2:W + 2])
    # and the second block = +1 moves along the height
    out = oracle.dcnv4_forward(x, _om(z, dx, m), G=G, K=K, pad=1)
    np.testing.assert_array_equal(out, xp[:, 2:H + 2, 1:W + 1])


def test_half_integer_offsets_average_two_neighbours():
    rng = np.random.default_rng(2)
    N, H, W, C, G, K = 1, 5, 8, 3, 1, 1
    x = rng.standard_normal((N, H, W, C))
    z = np.zeros((N, H, W, G, 1))
    half = np.full_like(z, 0.5)
    m = np.ones_like(z)
    out = oracle.dcnv4_forward(x, _om(half, z, m), G=G, K=K)
    xp = np.concatenate([x, np.zeros((N, H, 1, C))], axis=2)
    np.testing.assert_allclose(out, 0.5 * (xp[:, :, :-1] + xp[:, :, 1:]), rtol=0, atol=1e-15)
    out = oracle.dcnv4_forward(x, _om(z, -half, m), G=G, K=K)
    xp = np.concatenate([np.zeros((N, 1, W, C)), x], axis=1)
    np.testing.assert_allclose(out, 0.5 * (xp[:, :-1] + xp[:, 1:]), rtol=0, atol=1e-15)


def test_partition_of_unity_interior():
    rng = np.random.default_rng(3)
    N, H, W, C, G, K = 1, 12, 12, 4, 2, 3
    KK = K * K
    c = 1.75
    x = np.full((N, H, W, C), c)
    off = rng.uniform(-1.5, 1.5, size=(N, H, W, G, 2 * KK))
    m = rng.standard_normal((N, H, W, G, KK))
    out = oracle.dcnv4_forward(x, np.concatenate([off, m], -1), G=G, K=K, pad=1)
    expect = c * m.sum(-1)  # [N,H,W,G]
    inner = (slice(None), slice(3, H - 3), slice(3, W - 3))
    got = out.reshape(N, H, W, G, C // G)[inner]
    np.testing.assert_allclose(got, np.broadcast_to(expect[inner][..., None], got.shape),
                               rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------- brute force ---

def _brute_integer(x, om, G, K, stride, pad, dil):
    """Integer offsets: every sample is exactly one pixel; gather with numpy."""
    N, H, W, C = x.shape
    _, Hout, Wout, _, R = om.shape
    KK = K * K
    Cg = C // G
    B = 64
    xp = np.zeros((N, H + 2 * B, W + 2 * B, C))
    xp[:, B:B + H, B:B + W] = x
    out = np.zeros((N, Hout, Wout, C))
    ho = np.arange(Hout)[:, None]
    wo = np.arange(Wout)[None, :]
    for n in range(N):
        for g in range(G):
            for k in range(KK):
                ky, kx = divmod(k, K)
                yy = ho * stride - pad + ky * dil + om[n, :, :, g, KK + k].astype(np.int64)
                xx = wo * stride - pad + kx * dil + om[n, :, :, g, k].astype(np.int64)
                vals = xp[n, yy + B, xx + B][..., g * Cg:(g + 1) * Cg]
                out[n, :, :, g * Cg:(g + 1) * Cg] += om[n, :, :, g, 2 * KK + k][..., None] * vals
    return out


@pytest.mark.parametrize("N,H,W,C,G,K,stride,pad,dil", [
    (2, 7, 9, 8, 2, 3, 1, 1, 1),
    (1, 10, 6, 6, 3, 3, 2, 1, 1),
    (1, 9, 9, 4, 1, 3, 1, 2, 2),
    (2, 8, 8, 10, 5, 5, 1, 2, 1),
    (1, 6, 7, 3, 3, 1, 1, 0, 1),
])
def test_integer_offsets_match_bruteforce_gather(N, H, W, C, G, K, stride, pad, dil):
    rng = np.random.default_rng(H * 100 + W)
    Hout, Wout = _osz(H, K, stride, pad, dil), _osz(W, K, stride, pad, dil)
    KK = K * K
    off = rng.integers(-3, 4, size=(N, Hout, Wout, G, 2 * KK)).astype(np.float64)
    m = rng.standard_normal((N, Hout, Wout, G, KK))
    x = rng.standard_normal((N, H, W, C))
    om = np.concatenate([off, m], -1)
    out = oracle.dcnv4_forward(x, om, G=G, K=K, stride=stride, pad=pad, dilation=dil)
    np.testing.assert_allclose(out, _brute_integer(x, om, G, K, stride, pad, dil), rtol=0, atol=1e-13)


def test_zero_offsets_are_a_grouped_conv_with_per_pixel_weights():
    """Zero offsets reduce the op to a grouped KxK correlation whose weights
    change per pixel: checked against torch unfold (im2col) in fp64."""
    rng = np.random.default_rng(5)
    N, H, W, C, G, K, stride, pad, dil = 2, 9, 10, 12, 4, 3, 2, 1, 2
    Hout, Wout = _osz(H, K, stride, pad, dil), _osz(W, K, stride, pad, dil)
    KK = K * K
    x = rng.standard_normal((N, H, W, C))
    m = rng.standard_normal((N, Hout, Wout, G, KK))
    om = np.concatenate([np.zeros((N, Hout, Wout, G, 2 * KK)), m], -1)
    out = oracle.dcnv4_forward(x, om, G=G, K=K, stride=stride, pad=pad, dilation=dil)
    cols = torch.nn.functional.unfold(torch.from_numpy(x).permute(0, 3, 1, 2), K, dilation=dil,
                                      padding=pad, stride=stride)  # [N, C*KK, L]
    cols = cols.reshape(N, G, C // G, KK, Hout, Wout).numpy()
    ref = np.einsum("ngckhw,nhwgk->nhwgc", cols, m).reshape(N, Hout, Wout, C)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


# ------------------------------------------------------------- library routine ---

def _grid_sample_ref(x, om, G, K, stride, pad, dil, scale):
    """sum_k m_k * bilinear(x_g, p0_k + s*d_k) with torch grid_sample (fp64,
    zero padding, align_corners=True maps pixel p to 2p/(size-1)-1)."""
    N, H, W, C = x.shape
    _, Hout, Wout, _, _ = om.shape
    KK = K * K
    Cg = C // G
    xt = torch.from_numpy(x).permute(0, 3, 1, 2)  # N,C,H,W
    out = torch.zeros((N, C, Hout, Wout), dtype=torch.float64)
    ho = torch.arange(Hout, dtype=torch.float64)[:, None]
    wo = torch.arange(Wout, dtype=torch.float64)[None, :]
    omt = torch.from_numpy(om)
    for g in range(G):
        xg = xt[:, g * Cg:(g + 1) * Cg]
        for k in range(KK):
            ky, kx = divmod(k, K)
            # the scaled offset is an fp32 product (exact for the scales used here)
            dx = (omt[..., g, k].float() * np.float32(scale)).double()
            dy = (omt[..., g, KK + k].float() * np.float32(scale)).double()
            py = ho * stride - pad + ky * dil + dy
            px = wo * stride - pad + kx * dil + dx
            grid = torch.stack([2 * px / (W - 1) - 1, 2 * py / (H - 1) - 1], dim=-1)
            s = torch.nn.functional.grid_sample(xg, grid, mode="bilinear", padding_mode="zeros",
                                                align_corners=True)
            out[:, g * Cg:(g + 1) * Cg] += omt[..., g, 2 * KK + k][:, None] * s
    return out.permute(0, 2, 3, 1).numpy()


@pytest.mark.parametrize("N,H,W,C,G,K,stride,pad,dil,scale,spread", [
    (2, 8, 8, 16, 2, 3, 1, 1, 1, 1.0, 2.0),
    (1, 11, 7, 6, 3, 3, 2, 1, 1, 0.5, 3.0),
    (1, 12, 12, 8, 2, 3, 1, 1, 2, 1.0, 8.0),
    (1, 9, 9, 10, 2, 5, 1, 2, 1, 0.25, 6.0),
    (2, 5, 6, 4, 4, 1, 1, 0, 1, 1.0, 1.0),
])
def test_fractional_offsets_match_grid_sample(N, H, W, C, G, K, stride, pad, dil, scale, spread):
    rng = np.random.default_rng(H * 7 + K)
    Hout, Wout = _osz(H, K, stride, pad, dil), _osz(W, K, stride, pad, dil)
    KK = K * K
    x = rng.standard_normal((N, H, W, C))
    off = rng.uniform(-spread, spread, size=(N, Hout, Wout, G, 2 * KK)).astype(np.float32).astype(np.float64)
    m = rng.standard_normal((N, Hout, Wout, G, KK))
    om = np.concatenate([off, m], -1)
    out = oracle.dcnv4_forward(x, om, G=G, K=K, stride=stride, pad=pad, dilation=dil, offset_scale=scale)
    ref = _grid_sample_ref(x, om, G, K, stride, pad, dil, scale)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12 * max(1.0, np.abs(ref).max()))


# ----------------------------------------------------------------- invariants ---

def test_linear_in_mask_and_in_x():
    rng = np.random.default_rng(6)
    N, H, W, C, G, K = 1, 7, 7, 6, 2, 3
    KK = K * K
    x = rng.standard_normal((N, H, W, C))
    off = rng.uniform(-2, 2, size=(N, H, W, G, 2 * KK))
    m1 = rng.standard_normal((N, H, W, G, KK))
    m2 = rng.standard_normal((N, H, W, G, KK))
    f = lambda xx, mm: oracle.dcnv4_forward(xx, np.concatenate([off, mm], -1), G=G, K=K, pad=1)
    np.testing.assert_allclose(f(x, m1 + m2), f(x, m1) + f(x, m2), rtol=0, atol=1e-12)
    np.testing.assert_array_equal(f(x, 4.0 * m1), 4.0 * f(x, m1))
    np.testing.assert_array_equal(f(x / 4.0, 4.0 * m1), f(x, m1))
    np.testing.assert_allclose(f(2.0 * x - 1.0, m1), 2.0 * f(x, m1) - f(np.ones_like(x), m1),
                               rtol=0, atol=1e-12)


def test_out_of_bounds_and_non_finite_offsets_give_zero():
    rng = np.random.default_rng(7)
    N, H, W, C, G, K = 1, 6, 5, 4, 2, 3
    KK = K * K
    x = rng.standard_normal((N, H, W, C))
    m = rng.standard_normal((N, H, W, G, KK))
    far = float(H + W + 4)
    for dx, dy in [(far, 0.0), (-far, 0.0), (0.0, far), (0.0, -far), (1e30, 1e30), (-3e38, 0.0),
                   (math.inf, 0.0), (0.0, -math.inf), (math.nan, 0.0), (0.0, math.nan)]:
        off = np.concatenate([np.full((N, H, W, G, KK), dx), np.full((N, H, W, G, KK), dy)], -1)
        out = oracle.dcnv4_forward(x, np.concatenate([off, m], -1), G=G, K=K, pad=1)
        np.testing.assert_array_equal(out, np.zeros_like(out))
    # half a pixel off the top: only the first row of corners survives, weighted by 1 - fy = 0.5
    off = np.concatenate([np.zeros((N, H, W, G, KK)), np.full((N, H, W, G, KK), -0.5)], -1)
    mm = np.zeros_like(m)
    mm[..., 4] = 1.0
    out = oracle.dcnv4_forward(x, np.concatenate([off, mm], -1), G=G, K=K, pad=1)
    np.testing.assert_allclose(out[:, 0], 0.5 * x[:, 0], rtol=0, atol=1e-15)


def test_nan_in_x_reaches_only_samples_that_touch_it():
    N, H, W, C, G, K = 1, 6, 6, 2, 1, 1
    x = np.ones((N, H, W, C))
    x[0, 2, 3, :] = np.nan
    om = np.zeros((N, H, W, G, 3))
    om[..., 2] = 1.0
    out = oracle.dcnv4_forward(x, om, G=G, K=K)
    nan = np.isnan(out[0, :, :, 0])
    # with zero offsets the sample at (ho, wo) has corners (ho..ho+1, wo..wo+1), all
    # in bounds ones counted (weight 0 or not), so the NaN at (2, 3) reaches the four
    # outputs whose corner square contains it
    expect = np.zeros((H, W), bool)
    expect[1:3, 2:4] = True
    np.testing.assert_array_equal(nan, expect)
    assert np.isfinite(np.delete(out.reshape(-1, C), [1 * W + 2, 1 * W + 3, 2 * W + 2, 2 * W + 3], 0)).all()


def test_identical_group_records_equal_one_group():
    rng = np.random.default_rng(8)
    N, H, W, C, G, K = 2, 6, 7, 12, 3, 3
    KK = K * K
    x = rng.standard_normal((N, H, W, C))
    rec = np.concatenate([rng.uniform(-2, 2, (N, H, W, 1, 2 * KK)), rng.standard_normal((N, H, W, 1, KK))], -1)
    out_g = oracle.dcnv4_forward(x, np.repeat(rec, G, axis=3), G=G, K=K, pad=1)
    out_1 = oracle.dcnv4_forward(x, rec, G=1, K=K, pad=1)
    np.testing.assert_array_equal(out_g, out_1)


def test_translation_equivariance_interior():
    rng = np.random.default_rng(9)
    N, H, W, C, G, K = 1, 16, 16, 4, 2, 3
    KK = K * K
    x = rng.standard_normal((N, H, W, C))
    om = np.concatenate([rng.uniform(-1.5, 1.5, (N, H, W, G, 2 * KK)), rng.standard_normal((N, H, W, G, KK))], -1)
    ty, tx = 2, 3
    out = oracle.dcnv4_forward(x, om, G=G, K=K, pad=1)
    out_s = oracle.dcnv4_forward(np.roll(x, (ty, tx), axis=(1, 2)), np.roll(om, (ty, tx), axis=(1, 2)),
                                 G=G, K=K, pad=1)
    r = slice(4, H - 8)
    np.testing.assert_array_equal(out_s[:, 4 + ty:H - 8 + ty, 4 + tx:W - 8 + tx], out[:, r, r])


def test_sampling_index_for_integer_offsets_is_the_target_pixel():
    rng = np.random.default_rng(10)
    N, H, W, G, K, stride, pad, dil = 1, 7, 9, 2, 3, 1, 1, 2
    Hout, Wout = _osz(H, K, stride, pad, dil), _osz(W, K, stride, pad, dil)
    KK = K * K
    off = rng.integers(-5, 6, size=(N, Hout, Wout, G, 2 * KK)).astype(np.float64)
    om = np.concatenate([off, np.ones((N, Hout, Wout, G, KK))], -1)
    corner, valid = oracle.sampling_index(om, H, W, G, K, stride, pad, dil)
    for ho in range(Hout):
        for wo in range(Wout):
            for g in range(G):
                for k in range(KK):
                    ky, kx = divmod(k, K)
                    y = ho * stride - pad + ky * dil + int(off[0, ho, wo, g, KK + k])
                    x_ = wo * stride - pad + kx * dil + int(off[0, ho, wo, g, k])
                    inside = 0 <= y < H and 0 <= x_ < W
                    assert bool(valid[0, ho, wo, g, k] & 1) == inside
                    if valid[0, ho, wo, g, k]:
                        assert tuple(corner[0, ho, wo, g, k]) == (y, x_)


def test_output_size_matches_convolution_arithmetic():
    # torch's convolution output size is an independent statement of the formula
    for H, K, s, p, d in [(56, 3, 1, 1, 1), (256, 3, 1, 1, 2), (14, 3, 2, 1, 1), (9, 5, 3, 2, 2), (4, 2, 2, 0, 2)]:
        t = torch.nn.functional.conv2d(torch.zeros(1, 1, H, H), torch.zeros(1, 1, K, K), stride=s,
                                       padding=p, dilation=d)
        assert oracle.output_size(H, K, s, p, d) == t.shape[-1]
    assert oracle.output_size(2, 5, 1, 0, 1) <= 0


@pytest.mark.parametrize("name", ["tiny_f32", "stage3_f16", "sd_latent_f16", "highres_bf16"])
def test_parallel_oracle_gives_the_same_bits(name):
    """The all-core oracle (OpenMP over output rows, used to time the CPU
    baseline) computes every element with the same code in the same order as
    the single-thread one: the results are identical."""
    w = WORKLOADS[name]
    x, om = workload_inputs(w)
    xd, omd = x.double().numpy(), om.double().numpy()
    n1 = min(w.N, 2)
    a = oracle.dcnv4_forward(xd, omd, **w.kwargs(), n_begin=0, n_end=n1)
    b = oracle.dcnv4_forward(xd, omd, **w.kwargs(), n_begin=0, n_end=n1, threads=0)
    c = oracle.dcnv4_forward(xd, omd, **w.kwargs(), n_begin=0, n_end=n1, threads=3)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(a, c)
