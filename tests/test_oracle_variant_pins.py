"""Pins for the oracle's forward variants (softmax over the masks, removal of
the centre point, centre feature scaling), each against a statement that does
not reuse the variant code: scipy's softmax and expit, a full K*K record built
in numpy with the centre point switched off, numpy indexing for the centre
feature, closed forms at gate 0 and at saturation, and the identity case."""
import numpy as np
import pytest
from scipy.special import expit, softmax

import oracle


def _osz(n, K, s, p, d):
    return (n + 2 * p - d * (K - 1) - 1) // s + 1


def _case(seed, N, H, W, C, G, K, P, stride=1, pad=1, dil=1, spread=2.0):
    rng = np.random.default_rng(seed)
    Ho, Wo = _osz(H, K, stride, pad, dil), _osz(W, K, stride, pad, dil)
    x = rng.standard_normal((N, H, W, C))
    off = rng.uniform(-spread, spread, size=(N, Ho, Wo, G, 2 * P))
    m = rng.standard_normal((N, Ho, Wo, G, P))
    return x, np.concatenate([off, m], -1), rng.standard_normal((N, Ho, Wo, G))


def _insert_centre(om_rc, K, centre_mask=0.0):
    """Full K*K record from a remove_center record: centre offsets 0, centre mask `centre_mask`."""
    KK, P = K * K, K * K - 1
    c = (KK - 1) // 2
    dx, dy, m = om_rc[..., :P], om_rc[..., P:2 * P], om_rc[..., 2 * P:]
    ins = lambda a, v: np.concatenate([a[..., :c], np.full(a[..., :1].shape, v), a[..., c:]], -1)
    return np.concatenate([ins(dx, 0.0), ins(dy, 0.0), ins(m, centre_mask)], -1)


def _centre_feature(x, Ho, Wo, G, K, stride, pad, dil):
    N, H, W, C = x.shape
    xc = np.zeros((N, Ho, Wo, C))
    for ho in range(Ho):
        for wo in range(Wo):
            cy, cx = ho * stride - pad + (K // 2) * dil, wo * stride - pad + (K // 2) * dil
            if 0 <= cy < H and 0 <= cx < W:
                xc[:, ho, wo] = x[:, cy, cx]
    return xc


@pytest.mark.parametrize("shape", [(2, 7, 8, 8, 2, 3, 1, 1, 1), (1, 9, 9, 12, 3, 5, 1, 2, 1), (1, 10, 9, 6, 1, 3, 2, 1, 2)])
def test_softmax_variant_is_the_forward_with_softmaxed_masks(shape):
    N, H, W, C, G, K, s, p, d = shape
    KK = K * K
    x, om, _ = _case(1, N, H, W, C, G, K, KK, s, p, d)
    kw = dict(G=G, K=K, stride=s, pad=p, dilation=d)
    got = oracle.dcnv4_forward_variants(x, om, softmax=True, **kw)
    norm = om.copy()
    norm[..., 2 * KK:] = softmax(om[..., 2 * KK:], axis=-1)
    np.testing.assert_allclose(got, oracle.dcnv4_forward(x, norm, **kw), rtol=0, atol=1e-12)
    # softmax is invariant to a common shift of the masks
    shifted = om.copy()
    shifted[..., 2 * KK:] += 3.0
    np.testing.assert_allclose(oracle.dcnv4_forward_variants(x, shifted, softmax=True, **kw), got, rtol=0, atol=1e-12)


def test_softmax_with_equal_masks_is_the_mean_of_the_samples():
    N, H, W, C, G, K = 1, 6, 6, 4, 2, 3
    KK = K * K
    x, om, _ = _case(2, N, H, W, C, G, K, KK)
    om[..., 2 * KK:] = 0.7
    mean = om.copy()
    mean[..., 2 * KK:] = 1.0 / KK
    np.testing.assert_allclose(oracle.dcnv4_forward_variants(x, om, G=G, K=K, pad=1, softmax=True),
                               oracle.dcnv4_forward(x, mean, G=G, K=K, pad=1), rtol=0, atol=1e-13)


@pytest.mark.parametrize("K,pad,dil,stride", [(3, 1, 1, 1), (5, 2, 1, 1), (3, 2, 2, 1), (3, 1, 1, 2)])
def test_remove_center_equals_full_record_with_the_centre_switched_off(K, pad, dil, stride):
    N, H, W, C, G = 2, 9, 10, 8, 2
    P = K * K - 1
    x, om, _ = _case(3 + K, N, H, W, C, G, K, P, stride, pad, dil)
    kw = dict(G=G, K=K, stride=stride, pad=pad, dilation=dil)
    got = oracle.dcnv4_forward_variants(x, om, remove_center=True, **kw)
    np.testing.assert_array_equal(got, oracle.dcnv4_forward(x, _insert_centre(om, K), **kw))
    # with the softmax: the centre gets weight exp(-inf) = 0 in a K*K softmax
    gs = oracle.dcnv4_forward_variants(x, om, remove_center=True, softmax=True, **kw)
    full = _insert_centre(om, K, centre_mask=-np.inf)
    full[..., 2 * K * K:] = softmax(full[..., 2 * K * K:], axis=-1)
    np.testing.assert_allclose(gs, oracle.dcnv4_forward(x, full, **kw), rtol=0, atol=1e-12)


def test_remove_center_needs_an_odd_kernel_of_at_least_three():
    x = np.zeros((1, 6, 6, 4))
    for K, pad in ((2, 0), (4, 1), (1, 0)):
        P = K * K - 1
        Ho = _osz(6, K, 1, pad, 1)
        with pytest.raises(ValueError):
            oracle.dcnv4_forward_variants(x, np.zeros((1, Ho, Ho, 2, 3 * max(P, 1))), G=2, K=K, pad=pad,
                                          remove_center=True)


@pytest.mark.parametrize("K,stride,pad,dil", [(3, 1, 1, 1), (3, 2, 1, 1), (5, 1, 1, 2), (3, 1, 0, 1)])
def test_centre_scaling_blends_with_the_centre_feature(K, stride, pad, dil):
    N, H, W, C, G = 2, 9, 8, 12, 3
    KK = K * K
    x, om, z = _case(5, N, H, W, C, G, K, KK, stride, pad, dil)
    Ho, Wo = om.shape[1:3]
    kw = dict(G=G, K=K, stride=stride, pad=pad, dilation=dil)
    agg = oracle.dcnv4_forward(x, om, **kw)
    xc = _centre_feature(x, Ho, Wo, G, K, stride, pad, dil)
    s = np.repeat(expit(z), C // G, axis=-1)
    got = oracle.dcnv4_forward_variants(x, om, center_logit=z, **kw)
    np.testing.assert_allclose(got, (1 - s) * agg + s * xc, rtol=0, atol=1e-12)
    # gate 0 -> the mean of the two; saturated gates -> one side
    half = oracle.dcnv4_forward_variants(x, om, center_logit=np.zeros_like(z), **kw)
    np.testing.assert_allclose(half, 0.5 * agg + 0.5 * xc, rtol=0, atol=1e-12)
    np.testing.assert_allclose(oracle.dcnv4_forward_variants(x, om, center_logit=np.full_like(z, -60.0), **kw),
                               agg, rtol=0, atol=1e-12)
    np.testing.assert_allclose(oracle.dcnv4_forward_variants(x, om, center_logit=np.full_like(z, 60.0), **kw),
                               xc, rtol=0, atol=1e-12)


def test_identity_stays_identity_under_centre_scaling():
    N, H, W, C, G, K = 1, 7, 6, 8, 2, 3
    KK = K * K
    x = np.random.default_rng(9).standard_normal((N, H, W, C))
    om = np.zeros((N, H, W, G, 3 * KK))
    om[..., 2 * KK + (KK - 1) // 2] = 1.0
    z = np.random.default_rng(10).standard_normal((N, H, W, G))
    # (1 - s) x + s x: equal to x up to one rounding of each term
    np.testing.assert_allclose(oracle.dcnv4_forward_variants(x, om, G=G, K=K, pad=1, center_logit=z), x,
                               rtol=1e-15, atol=0)
