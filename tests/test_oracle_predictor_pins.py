"""Pins for the oracle's offset/mask predictor step (1x1 projection + repacking
into offset_mask records): numpy's matmul followed by the reshapes of the
pages' listings (offsets as (G, 2, P), masks as (G, P)), a hand case, and the
round trip through the oracle's forward."""
import numpy as np
import pytest

import oracle


@pytest.mark.parametrize("C,G,P", [(64, 4, 9), (32, 2, 8), (16, 1, 1), (128, 8, 9)])
def test_predictor_is_matmul_then_the_listing_reshapes(C, G, P):
    rng = np.random.default_rng(C + G + P)
    M = 37
    y = rng.standard_normal((M, C))
    w = rng.standard_normal((3 * G * P, C))
    b = rng.standard_normal(3 * G * P)
    params = y @ w.T + b                                   # [M, 3GP]
    off = params[:, :2 * G * P].reshape(M, G, 2, P)        # offset.reshape(N, G, 2, P, ...)
    msk = params[:, 2 * G * P:].reshape(M, G, P)           # mask.reshape(N, G, P, ...)
    want = np.concatenate([off[:, :, 0], off[:, :, 1], msk], axis=-1)
    got = oracle.dcnv4_predictor(y, w, b, G=G, P=P)
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-12)
    np.testing.assert_allclose(oracle.dcnv4_predictor(y.reshape(1, M, 1, C), w, None, G=G, P=P)[0, :, 0],
                               want - np.concatenate([b[:2 * G * P].reshape(G, 2, P)[:, 0],
                                                      b[:2 * G * P].reshape(G, 2, P)[:, 1],
                                                      b[2 * G * P:].reshape(G, P)], -1), rtol=1e-12, atol=1e-12)


def test_hand_case_two_groups_one_point():
    # G = 2, P = 1: channels o = [g0 dx, g0 dy, g1 dx, g1 dy, g0 m, g1 m]; C = 2, y = (1, 2)
    w = np.array([[1, 0], [0, 1], [1, 1], [2, 0], [0, 3], [1, -1]], dtype=float)
    b = np.array([0.5, 0, 0, 0, 0, 10], dtype=float)
    rec = oracle.dcnv4_predictor(np.array([[1.0, 2.0]]), w, b, G=2, P=1)
    # group 0: dx = 1 + 0.5, dy = 2, m = 6; group 1: dx = 3, dy = 2, m = 1 - 2 + 10
    np.testing.assert_array_equal(rec, [[[1.5, 2.0, 6.0], [3.0, 2.0, 9.0]]])


def test_predicted_record_drives_the_forward():
    # zero weights, bias = (zero offsets, one-hot centre mask): the forward is the identity
    G, K, C = 2, 3, 8
    P = K * K
    bias = np.zeros(3 * G * P)
    bias[2 * G * P + 0 * P + 4] = 1.0
    bias[2 * G * P + 1 * P + 4] = 1.0
    x = np.random.default_rng(1).standard_normal((1, 5, 6, C))
    rec = oracle.dcnv4_predictor(x, np.zeros((3 * G * P, C)), bias, G=G, P=P)
    np.testing.assert_array_equal(oracle.dcnv4_forward(x, rec, G=G, K=K, pad=1), x)
