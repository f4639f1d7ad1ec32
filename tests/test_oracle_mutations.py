"""Plant plausible mistakes in the oracle and check that the pins catch them.

Each mutant replaces one step of ``oracle.favor`` (a dropped term, a wrong
scale, a wrong index, a wrong sign, a transposed operand) for the duration of
one test.  The unmutated oracle must pass every check; each mutant must fail
at least one.  The checks are fast versions of the pins in
``test_oracle_favor.py`` and ``test_oracle_features.py``.
"""
import math

import numpy as np
import pytest
from scipy import special

from oracle import favor


def check_unbiased():
    d = 16
    rng = np.random.default_rng(7)
    q = rng.standard_normal(d) * 0.45
    k = rng.standard_normal(d) * 0.45
    est = []
    for s in range(600):
        W = favor.make_features(20_000 + s, d, d)
        pq, _ = favor.query_features(q[None, :], W, stabilise=False)
        pk, _ = favor.key_features(k[None, :], W, stabilise=False)
        est.append(float(pq[0] @ pk[0]))
    est = np.array(est)
    target = math.exp(float(q @ k) / math.sqrt(d))
    return abs(est.mean() - target) < 4 * est.std(ddof=1) / math.sqrt(est.size)


def check_stabilisers_cancel():
    rng = np.random.default_rng(3)
    Q = rng.standard_normal((1, 2, 30, 16)) * 0.8
    K = rng.standard_normal((1, 1, 30, 16)) * 0.8
    V = rng.standard_normal((1, 1, 30, 16))
    W = favor.make_features(4, 32, 16)
    a = favor.favor_attention(Q, K, V, W, stabilise=True)
    b = favor.favor_attention(Q, K, V, W, stabilise=False)
    return np.allclose(a, b, rtol=1e-12, atol=1e-13)


def check_large_inputs_finite():
    rng = np.random.default_rng(4)
    Q = rng.standard_normal((1, 1, 20, 16)) * 25
    K = rng.standard_normal((1, 1, 20, 16)) * 25
    V = rng.standard_normal((1, 1, 20, 16))
    with np.errstate(all="ignore"):
        out = favor.favor_attention(Q, K, V, favor.make_features(5, 32, 16))
    return bool(np.all(np.isfinite(out)))


def check_converges_to_softmax():
    d, L = 16, 16
    rng = np.random.default_rng(12)
    Q = rng.standard_normal((1, 4, L, d)) * 0.25
    K = rng.standard_normal((1, 2, L, d)) * 0.25
    V = rng.standard_normal((1, 2, L, d))
    exact = favor.softmax_attention(Q, K, V)
    e = [np.abs(favor.favor_attention(Q, K, V, favor.make_features(s, 4096, d)) - exact).max()
         for s in range(4)]
    return float(np.mean(e)) < 0.03


def check_linear_equals_quadratic():
    rng = np.random.default_rng(2)
    Q = rng.standard_normal((1, 2, 20, 16)) * 0.7
    K = rng.standard_normal((1, 1, 20, 16)) * 0.7
    V = rng.standard_normal((1, 1, 20, 16))
    W = favor.make_features(3, 32, 16)
    return np.allclose(favor.favor_attention(Q, K, V, W), favor.favor_quadratic(Q, K, V, W),
                       rtol=1e-12, atol=1e-13)


def check_chi_norms():
    d = 64
    W = favor.make_features(11, 64 * 16, d)
    r = np.sqrt(np.sum(W * W, axis=1))
    mu = math.sqrt(2.0) * math.exp(special.gammaln((d + 1) / 2) - special.gammaln(d / 2))
    return abs(r.mean() - mu) < 4 * math.sqrt(d - mu * mu) / math.sqrt(r.size) and r.std() > 0.1


def check_convex_hull():
    rng = np.random.default_rng(5)
    Q = rng.standard_normal((1, 2, 40, 16))
    K = rng.standard_normal((1, 2, 40, 16))
    V = rng.standard_normal((1, 2, 40, 16))
    out = favor.favor_attention(Q, K, V, favor.make_features(6, 32, 16))
    return all(np.all(out[0, h] >= V[0, h].min(0) - 1e-12) and np.all(out[0, h] <= V[0, h].max(0) + 1e-12)
               for h in range(2))


CHECKS = [check_unbiased, check_stabilisers_cancel, check_large_inputs_finite,
          check_converges_to_softmax, check_linear_equals_quadratic, check_chi_norms,
          check_convex_hull]


def _all_pass():
    results = {}
    for c in CHECKS:
        try:
            results[c.__name__] = bool(c())
        except Exception:  # a mutant may also break shapes
            results[c.__name__] = False
    return results


# ---- mutants ---------------------------------------------------------------
def m_drop_norm_term(Xs, W):
    return Xs @ np.asarray(W, dtype=np.float64).T


def m_norm_term_sign(Xs, W):
    W = np.asarray(W, dtype=np.float64)
    return Xs @ W.T + 0.5 * np.sum(Xs * Xs, axis=1, keepdims=True)


def m_transposed_w(Xs, W):
    W = np.asarray(W, dtype=np.float64)
    return Xs @ W - 0.5 * np.sum(Xs * Xs, axis=1, keepdims=True)


def m_scale_sqrt_d(X):
    X = np.asarray(X, dtype=np.float64)
    return X * X.shape[-1] ** -0.5


def m_per_key_stabiliser(K, W, stabilise=True):
    u = favor.exponents(favor.scale_inputs(K), W)
    c = u.max(axis=1, keepdims=True) if stabilise else 0.0
    return np.exp(u - c) / math.sqrt(W.shape[0]), c


def m_stabiliser_sign(K, W, stabilise=True):
    u = favor.exponents(favor.scale_inputs(K), W)
    c = float(u.max()) if stabilise else 0.0
    return np.exp(u + c) / math.sqrt(W.shape[0]), c


def m_kv_head_modulo(Q, K, V, W, stabilise=True):
    B, H, L, d = Q.shape
    Hkv = K.shape[1]
    out = np.empty(Q.shape)
    for b in range(B):
        for h in range(H):
            S, _ = favor.key_state(K[b, h % Hkv], V[b, h % Hkv], W, stabilise)
            out[b, h] = favor.query_output(Q[b, h], W, S, stabilise)
    return out


def m_unit_norm_rows(seed, m, d, orthogonal=True):
    W = _orig_make_features(seed, m, d, orthogonal)
    return W / np.linalg.norm(W, axis=1, keepdims=True) * math.sqrt(d)


def m_key_state_without_ones(K, V, W, stabilise=True):
    phik, c = favor.key_features(K, W, stabilise)
    V = np.asarray(V, dtype=np.float64)
    S = phik.T @ np.concatenate([V, V[:, :1]], axis=1)
    return S, c


_orig_make_features = favor.make_features

MUTANTS = {
    "drop -|x|^2/2": ("exponents", m_drop_norm_term),
    "+|x|^2/2": ("exponents", m_norm_term_sign),
    "W not transposed": ("exponents", m_transposed_w),
    "scale d^-1/2": ("scale_inputs", m_scale_sqrt_d),
    "per-key stabiliser": ("key_features", m_per_key_stabiliser),
    "stabiliser added": ("key_features", m_stabiliser_sign),
    "kv head h % Hkv": ("favor_attention", m_kv_head_modulo),
    "norms not resampled": ("make_features", m_unit_norm_rows),
    "ones column replaced": ("key_state", m_key_state_without_ones),
}


def test_unmutated_oracle_passes_every_check():
    res = _all_pass()
    assert all(res.values()), res


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(favor, attr, fn)
    res = _all_pass()
    assert not all(res.values()), f"mutant '{name}' passed every check: {res}"
