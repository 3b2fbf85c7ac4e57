"""Pins for the oracle's backward of the forward variants: without flags it is
the plain backward; without the centre point it is the plain backward of the
record with the centre switched off; for every flag set the adjoint identity in
x holds (the variants stay linear in x), central differences of the variants'
forward match the offset, mask and gate gradients, and softmax mask gradients
sum to zero per unit (the softmax ignores a common shift)."""
import numpy as np
import pytest

import oracle

FLAGS = [dict(), dict(softmax=True), dict(remove_center=True), dict(center=True),
         dict(softmax=True, remove_center=True, center=True)]


def _case(seed, N=1, H=6, W=7, C=6, G=2, K=3, P=None, grid=True):
    rng = np.random.default_rng(seed)
    P = K * K if P is None else P
    x = rng.standard_normal((N, H, W, C))
    if grid:   # offsets on a 1/64 grid, fractional parts in [1/4, 3/4]: exact central differences
        off = (rng.integers(-2, 3, size=(N, H, W, G, 2 * P)) + rng.integers(16, 49, size=(N, H, W, G, 2 * P)) / 64.0)
    else:
        off = rng.uniform(-2, 2, size=(N, H, W, G, 2 * P))
    m = rng.standard_normal((N, H, W, G, P))
    g = rng.standard_normal((N, H, W, C))
    z = rng.standard_normal((N, H, W, G))
    return x, np.concatenate([off, m], -1), g, z


def _kw(f):
    return dict(softmax=f.get("softmax", False), remove_center=f.get("remove_center", False))


def test_no_flags_is_the_plain_backward():
    x, om, g, _ = _case(1)
    a = oracle.dcnv4_backward(x, om, g, G=2, K=3, pad=1)
    b = oracle.dcnv4_backward_variants(x, om, g, G=2, K=3, pad=1)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
    assert b[2] is None


def test_remove_center_is_the_plain_backward_with_the_centre_switched_off():
    K, P = 3, 8
    x, om, g, _ = _case(2, P=P)
    c = (K * K - 1) // 2
    ins = lambda a, v: np.concatenate([a[..., :c], np.full(a[..., :1].shape, v), a[..., c:]], -1)
    full = np.concatenate([ins(om[..., :P], 0.0), ins(om[..., P:2 * P], 0.0), ins(om[..., 2 * P:], 0.0)], -1)
    gx_f, gom_f = oracle.dcnv4_backward(x, full, g, G=2, K=K, pad=1)
    gx, gom, _ = oracle.dcnv4_backward_variants(x, om, g, G=2, K=K, pad=1, remove_center=True)
    np.testing.assert_array_equal(gx, gx_f)
    keep = [i for i in range(3 * K * K) if i % (K * K) != c]
    np.testing.assert_array_equal(gom, gom_f[..., keep])


@pytest.mark.parametrize("f", FLAGS, ids=lambda f: "-".join(sorted(f)) or "none")
def test_adjoint_in_x(f):
    P = 8 if f.get("remove_center") else 9
    x, om, g, z = _case(3, P=P, grid=False)
    zz = z if f.get("center") else None
    out = oracle.dcnv4_forward_variants(x, om, G=2, K=3, pad=1, center_logit=zz, **_kw(f))
    gx, _, _ = oracle.dcnv4_backward_variants(x, om, g, G=2, K=3, pad=1, center_logit=zz, **_kw(f))
    lhs, rhs = float(np.sum(out * g)), float(np.sum(x * gx))
    assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs))


@pytest.mark.parametrize("f", FLAGS, ids=lambda f: "-".join(sorted(f)) or "none")
def test_central_differences(f):
    P = 8 if f.get("remove_center") else 9
    x, om, g, z = _case(4, P=P)
    zz = z if f.get("center") else None
    kw = dict(G=2, K=3, pad=1, **_kw(f))
    loss = lambda o, zv: float(np.sum(oracle.dcnv4_forward_variants(x, o, center_logit=zv, **kw) * g))
    _, gom, gz = oracle.dcnv4_backward_variants(x, om, g, center_logit=zz, **kw)
    # offsets: exact (the sample stays in its cell); masks: softmax is smooth, O(h^2) error
    for idx, h, tol in [((0, 2, 3, 1, 1), 2.0 ** -10, 1e-9), ((0, 4, 5, 0, P + 3), 2.0 ** -10, 1e-9),
                        ((0, 1, 2, 1, 2 * P + 2), 1e-5, 1e-7), ((0, 5, 6, 0, 2 * P + P - 1), 1e-5, 1e-7)]:
        a, b = om.copy(), om.copy()
        a[idx] += h
        b[idx] -= h
        fd = (loss(a, zz) - loss(b, zz)) / (2 * h)
        assert abs(fd - gom[idx]) <= tol * max(1.0, abs(fd)), (idx, fd, gom[idx])
    if zz is not None:
        for idx in [(0, 0, 0, 0), (0, 3, 4, 1)]:
            a, b = zz.copy(), zz.copy()
            a[idx] += 1e-5
            b[idx] -= 1e-5
            fd = (loss(om, a) - loss(om, b)) / 2e-5
            assert abs(fd - gz[idx]) <= 1e-7 * max(1.0, abs(fd)), (idx, fd, gz[idx])


def test_softmax_mask_gradients_sum_to_zero():
    x, om, g, _ = _case(5, grid=False)
    _, gom, _ = oracle.dcnv4_backward_variants(x, om, g, G=2, K=3, pad=1, softmax=True)
    np.testing.assert_allclose(gom[..., 18:].sum(-1), 0.0, atol=1e-12)
