"""Pins for the oracle's random-feature matrix W.

"Rethinking Attention with Performers" (Abstract; 제안 방법 / proposed method;
주요 결과 / main results) asks for orthogonal random features whose rows are
still Gaussian in distribution.  These tests check that against library
routines and closed forms, never against the oracle itself.
"""
import math

import numpy as np
import pytest
from scipy import special, stats

from oracle import favor, philox


def chi_mean(d):
    """E|g| for g ~ N(0, I_d): sqrt(2) Gamma((d+1)/2) / Gamma(d/2)."""
    return math.sqrt(2.0) * math.exp(special.gammaln((d + 1) / 2) - special.gammaln(d / 2))


def test_gram_schmidt_equals_sign_fixed_qr():
    # Rows orthonormalised first-to-last == (Q of QR(G^T), columns signed so R has a positive diagonal)^T
    rng = np.random.default_rng(3)
    for d in (4, 16, 64, 128):
        G = rng.standard_normal((d, d))
        q, r = np.linalg.qr(G.T)
        want = (q * np.sign(np.diag(r))[None, :]).T
        np.testing.assert_allclose(favor.gram_schmidt_rows(G), want, atol=1e-10)


@pytest.mark.parametrize("m,d", [(128, 64), (256, 64), (256, 128), (512, 64), (100, 16)])
def test_rows_orthogonal_within_blocks(m, d):
    W = favor.make_features(1, m, d, orthogonal=True)
    assert W.shape == (m, d)
    norms2 = np.sum(W * W, axis=1)
    for b in range(0, m, d):
        blk = W[b:b + d]
        gram = blk @ blk.T
        off = gram - np.diag(np.diag(gram))
        assert np.abs(off).max() <= 1e-12 * norms2.max()
        np.testing.assert_allclose(np.diag(gram), norms2[b:b + d], rtol=1e-14)
    if m > d:  # different blocks are independent, not orthogonal to each other
        assert np.abs(W[:d] @ W[d:2 * d].T).max() > 1.0


def test_row_norms_are_chi_distributed():
    d = 64
    W = favor.make_features(11, 64 * 64, d, orthogonal=True)
    r = np.sqrt(np.sum(W * W, axis=1))
    mu = chi_mean(d)
    sd = math.sqrt(d - mu * mu)
    assert abs(r.mean() - mu) < 4 * sd / math.sqrt(r.size)
    # chi(d) CDF: P(|g| <= x) = regularised lower gamma P(d/2, x^2/2)
    assert stats.kstest(r, lambda x: special.gammainc(d / 2, x * x / 2)).pvalue > 1e-3


def test_norms_come_from_their_own_stream():
    m, d = 32, 16
    W = favor.make_features(5, m, d, orthogonal=True)
    h = philox.normals(5, favor.TAG_NORMS, m * d).reshape(m, d)
    np.testing.assert_allclose(np.sqrt(np.sum(W * W, axis=1)), np.sqrt(np.sum(h * h, axis=1)), rtol=1e-13)


@pytest.mark.parametrize("orthogonal", [True, False])
def test_rows_have_identity_second_moment(orthogonal):
    # each row is marginally N(0, I_d): E[w w^T] = I and E[w] = 0
    m, d = 16 * 400, 16
    W = favor.make_features(21, m, d, orthogonal=orthogonal)
    C = W.T @ W / m
    assert np.abs(C - np.eye(d)).max() < 6 * math.sqrt(2.0 / m)
    assert np.abs(W.mean(axis=0)).max() < 6 / math.sqrt(m)


def test_iid_rows_are_the_raw_stream():
    m, d = 40, 16
    W = favor.make_features(9, m, d, orthogonal=False)
    g = philox.normals(9, favor.TAG_DIRECTIONS, 3 * d * d)[:m * d].reshape(m, d)
    np.testing.assert_array_equal(W, g)


def test_partial_last_block_keeps_leading_rows():
    d = 16
    full = favor.make_features(4, 48, d)
    part = favor.make_features(4, 40, d)
    # directions of the kept rows match; norms come from the first m norm vectors
    dirs_full = full / np.linalg.norm(full, axis=1, keepdims=True)
    dirs_part = part / np.linalg.norm(part, axis=1, keepdims=True)
    np.testing.assert_allclose(dirs_part, dirs_full[:40], atol=1e-13)


def test_exponent_bounded_by_half_squared_row_norm():
    # completing the square: w.x - |x|^2/2 = |w|^2/2 - |x - w|^2/2 <= |w|^2/2
    rng = np.random.default_rng(0)
    W = favor.make_features(1, 256, 64)
    X = rng.standard_normal((500, 64)) * rng.lognormal(0, 1.0, (500, 1)) * 3
    u = favor.exponents(favor.scale_inputs(X), W)
    assert np.all(u <= 0.5 * np.sum(W * W, axis=1)[None, :] + 1e-9)
