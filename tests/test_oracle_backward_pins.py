"""Pins for the fp64 oracle's backward pass, against checks that do not reuse
its code: a hand-derived case (tests/golden/hand_cases.json), the adjoint
identity <f(x), g> = <x, dL/dx> (the op is linear in x), Euler's identity
sum m dL/dm = <f, g> (it is linear in the masks), the per-point mask gradient
as the forward with one-hot masks, exact central differences for the offsets
(the sample is linear in the offset inside a pixel cell), a numpy scatter for
integer offsets, and zero gradients for samples outside the image."""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")


def _osz(n, K, s, p, d):
    return (n + 2 * p - d * (K - 1) - 1) // s + 1


def _rand_case(seed, N, H, W, C, G, K, stride=1, pad=1, dil=1, lo=-2.0, hi=2.0, grid=None):
    rng = np.random.default_rng(seed)
    Hout, Wout = _osz(H, K, stride, pad, dil), _osz(W, K, stride, pad, dil)
    KK = K * K
    x = rng.standard_normal((N, H, W, C))
    off = rng.uniform(lo, hi, size=(N, Hout, Wout, G, 2 * KK))
    if grid is not None:
        off = np.round(off * grid) / grid
    m = rng.standard_normal((N, Hout, Wout, G, KK))
    g = rng.standard_normal((N, Hout, Wout, C))
    return x, np.concatenate([off, m], -1), g


def test_golden_backward_case():
    case = json.load(open(GOLDEN))["cases"][0]
    bw = case["backward"]
    x = np.array(case["x"], dtype=np.float64)
    om = np.array(case["offset_mask"], dtype=np.float64)
    gx, gom = oracle.dcnv4_backward(x, om, np.array(bw["grad_out"]), G=1, K=1)
    np.testing.assert_array_equal(gx, np.array(bw["grad_x"]))
    np.testing.assert_array_equal(gom, np.array(bw["grad_offset_mask"]))


@pytest.mark.parametrize("shape", [(2, 7, 8, 8, 2, 3, 1, 1, 1), (1, 9, 6, 6, 3, 3, 2, 1, 1), (1, 8, 8, 4, 1, 3, 1, 2, 2),
                                   (2, 6, 7, 10, 5, 5, 1, 2, 1)])
def test_adjoint_identity_for_x(shape):
    N, H, W, C, G, K, s, p, d = shape
    x, om, g = _rand_case(sum(shape), N, H, W, C, G, K, s, p, d, -3, 3)
    kw = dict(G=G, K=K, stride=s, pad=p, dilation=d)
    out = oracle.dcnv4_forward(x, om, **kw)
    gx, _ = oracle.dcnv4_backward(x, om, g, **kw)
    lhs, rhs = float(np.sum(out * g)), float(np.sum(x * gx))
    assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs))


def test_euler_identity_for_masks_and_one_hot_masks():
    N, H, W, C, G, K = 1, 7, 7, 6, 2, 3
    KK = K * K
    x, om, g = _rand_case(3, N, H, W, C, G, K)
    out = oracle.dcnv4_forward(x, om, G=G, K=K, pad=1)
    _, gom = oracle.dcnv4_backward(x, om, g, G=G, K=K, pad=1)
    euler = float(np.sum(gom[..., 2 * KK:] * om[..., 2 * KK:]))
    assert abs(euler - float(np.sum(out * g))) <= 1e-12 * abs(euler)
    Cg = C // G
    for k in range(KK):
        one = om.copy()
        one[..., 2 * KK:] = 0.0
        one[..., 2 * KK + k] = 1.0
        sample = oracle.dcnv4_forward(x, one, G=G, K=K, pad=1).reshape(N, H, W, G, Cg)
        expect = np.sum(sample * g.reshape(N, H, W, G, Cg), axis=-1)
        np.testing.assert_allclose(gom[..., 2 * KK + k], expect, rtol=0, atol=1e-12)


@pytest.mark.parametrize("scale", [1.0, 0.5])
def test_offset_gradients_are_exact_central_differences(scale):
    # offsets on a 1/64 grid with fractional parts in [1/4, 3/4]: steps of 2^-10
    # stay inside the pixel cell and are exact in fp32, and the sample is linear
    # in the offset there, so the central difference is the derivative
    N, H, W, C, G, K = 1, 6, 7, 4, 2, 3
    KK = K * K
    rng = np.random.default_rng(11)
    Hout, Wout = H, W
    x = rng.standard_normal((N, H, W, C))
    base = rng.integers(-2, 3, size=(N, Hout, Wout, G, 2 * KK)).astype(np.float64)
    frac = rng.integers(16, 49, size=base.shape) / 64.0
    off = (base + frac) / scale
    m = rng.standard_normal((N, Hout, Wout, G, KK))
    om = np.concatenate([off, m], -1)
    g = rng.standard_normal((N, Hout, Wout, C))
    kw = dict(G=G, K=K, pad=1, offset_scale=scale)
    _, gom = oracle.dcnv4_backward(x, om, g, **kw)
    h = 2.0 ** -10 / scale
    probes = [(0, 0, 0, 0, 0), (0, 2, 3, 1, 4), (0, 5, 6, 0, 8), (0, 3, 1, 1, 2 + KK), (0, 4, 4, 0, 7 + KK),
              (0, 0, 6, 1, KK)]
    for idx in probes:
        p_, m_ = om.copy(), om.copy()
        p_[idx] += h
        m_[idx] -= h
        fd = (np.sum(oracle.dcnv4_forward(x, p_, **kw) * g) - np.sum(oracle.dcnv4_forward(x, m_, **kw) * g)) / (2 * h)
        assert abs(fd - gom[idx]) <= 1e-9 * max(1.0, abs(fd)), (idx, fd, gom[idx])


def test_integer_offsets_scatter_matches_numpy():
    N, H, W, C, G, K = 2, 6, 7, 6, 3, 3
    KK = K * K
    rng = np.random.default_rng(5)
    x = rng.standard_normal((N, H, W, C))
    off = rng.integers(-3, 4, size=(N, H, W, G, 2 * KK)).astype(np.float64)
    m = rng.standard_normal((N, H, W, G, KK))
    g = rng.standard_normal((N, H, W, C))
    gx, _ = oracle.dcnv4_backward(x, np.concatenate([off, m], -1), g, G=G, K=K, pad=1)
    ref = np.zeros_like(x)
    Cg = C // G
    for n in range(N):
        for ho in range(H):
            for wo in range(W):
                for gg in range(G):
                    for k in range(KK):
                        ky, kx = divmod(k, K)
                        y = ho - 1 + ky + int(off[n, ho, wo, gg, KK + k])
                        xx = wo - 1 + kx + int(off[n, ho, wo, gg, k])
                        if 0 <= y < H and 0 <= xx < W:
                            sl = slice(gg * Cg, (gg + 1) * Cg)
                            ref[n, y, xx, sl] += m[n, ho, wo, gg, k] * g[n, ho, wo, sl]
    np.testing.assert_allclose(gx, ref, rtol=0, atol=1e-12)


def test_samples_outside_give_zero_gradients():
    N, H, W, C, G, K = 1, 5, 5, 4, 2, 3
    KK = K * K
    x, om, g = _rand_case(8, N, H, W, C, G, K)
    for v in (float(H + W + 5), -1e30, math.inf, math.nan):
        bad = om.copy()
        bad[..., :KK] = v
        gx, gom = oracle.dcnv4_backward(x, bad, g, G=G, K=K, pad=1)
        assert not gx.any() and not gom.any()
