"""Pins for the oracle's FAVOR+ estimate.

"Rethinking Attention with Performers" states (Abstract; 주요 결과 / main
results) that the estimate is unbiased, converges to softmax attention and
costs linear space and time.  "Fast Transformer Decoding: One Write-Head is
All You Need" (提出的方法 / proposed method) fixes the shared K/V layout.  Each
test below checks one of those statements against mathematics or a library
routine, not against the oracle itself.
"""
import math

import numpy as np
import pytest
import torch

from oracle import favor


def _inputs(B, H, Hkv, L, d, scale=1.0, seed=0):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((B, H, L, d)) * scale
    K = rng.standard_normal((B, Hkv, L, d)) * scale
    V = rng.standard_normal((B, Hkv, L, d))
    return Q, K, V


def test_softmax_attention_matches_torch_sdpa_with_shared_kv():
    Q, K, V = _inputs(2, 6, 2, 33, 16, seed=1)
    G = 3
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q), torch.from_numpy(K).repeat_interleave(G, dim=1),
        torch.from_numpy(V).repeat_interleave(G, dim=1)).numpy()
    np.testing.assert_allclose(favor.softmax_attention(Q, K, V), want, rtol=1e-10, atol=1e-12)


def _mc_kernel_estimates(q, k, d, orthogonal, nseeds):
    """phi(q')^T phi(k') for m = d features, one W per seed (no stabiliser).

    Each phi carries 1/sqrt(m), so the product is (1/m) sum_r of the
    per-feature products, the estimator of exp(q.k / sqrt(d)).
    """
    est = np.empty(nseeds)
    for s in range(nseeds):
        W = favor.make_features(10_000 + s, d, d, orthogonal)
        pq, _ = favor.query_features(q[None, :], W, stabilise=False)
        pk, _ = favor.key_features(k[None, :], W, stabilise=False)
        est[s] = float(pq[0] @ pk[0])
    return est


@pytest.mark.parametrize("orthogonal", [True, False])
def test_feature_product_is_unbiased_for_softmax_kernel(orthogonal):
    d = 16
    rng = np.random.default_rng(7)
    q = rng.standard_normal(d) * 0.45
    k = rng.standard_normal(d) * 0.45
    est = _mc_kernel_estimates(q, k, d, orthogonal, 2000)
    target = math.exp(float(q @ k) / math.sqrt(d))
    se = est.std(ddof=1) / math.sqrt(est.size)
    assert abs(est.mean() - target) < 3.5 * se, (est.mean(), target, se)
    assert se < 0.05 * target  # the check has teeth


def test_orthogonal_features_lower_the_variance():
    # 주요 결과: orthogonal random features reduce the mean squared error
    d = 16
    rng = np.random.default_rng(8)
    q = rng.standard_normal(d) * 0.3
    k = rng.standard_normal(d) * 0.3
    target = math.exp(float(q @ k) / math.sqrt(d))
    n = 4000
    e_orf = (_mc_kernel_estimates(q, k, d, True, n) - target) ** 2
    e_iid = (_mc_kernel_estimates(q, k, d, False, n) - target) ** 2
    se = math.sqrt(e_orf.var() / n + e_iid.var() / n)
    assert e_iid.mean() - e_orf.mean() > 2.0 * se, (e_orf.mean(), e_iid.mean(), se)


def test_linear_order_equals_quadratic_form():
    Q, K, V = _inputs(1, 4, 2, 40, 16, scale=0.7, seed=2)
    W = favor.make_features(3, 48, 16)
    lin = favor.favor_attention(Q, K, V, W)
    quad = favor.favor_quadratic(Q, K, V, W)
    np.testing.assert_allclose(lin, quad, rtol=1e-12, atol=1e-13)


def test_stabilisers_cancel_exactly():
    Q, K, V = _inputs(2, 2, 1, 50, 16, scale=0.8, seed=3)
    W = favor.make_features(4, 64, 16)
    a = favor.favor_attention(Q, K, V, W, stabilise=True)
    b = favor.favor_attention(Q, K, V, W, stabilise=False)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


def test_stabilisers_keep_large_inputs_finite():
    # exponents near -900: without the stabiliser exp() underflows to 0 and the ratio is 0/0
    Q, K, V = _inputs(1, 1, 1, 20, 16, scale=25.0, seed=4)
    W = favor.make_features(5, 32, 16)
    out = favor.favor_attention(Q, K, V, W)
    assert np.all(np.isfinite(out))
    with np.errstate(invalid="ignore", divide="ignore"):
        raw = favor.favor_attention(Q, K, V, W, stabilise=False)
    assert not np.all(np.isfinite(raw))


def test_outputs_are_convex_combinations_of_values():
    Q, K, V = _inputs(2, 4, 2, 64, 16, seed=5)
    W = favor.make_features(6, 32, 16)
    out = favor.favor_attention(Q, K, V, W)
    G = 2
    for b in range(2):
        for h in range(4):
            lo = V[b, h // G].min(axis=0)
            hi = V[b, h // G].max(axis=0)
            assert np.all(out[b, h] >= lo - 1e-12) and np.all(out[b, h] <= hi + 1e-12)


def test_converges_to_softmax_attention_as_m_grows():
    # small-norm inputs (Q, K ~ N(0, 0.25^2)); shared K/V heads included
    d, L = 16, 16
    rng = np.random.default_rng(12)
    Q = rng.standard_normal((1, 4, L, d)) * 0.25
    K = rng.standard_normal((1, 2, L, d)) * 0.25
    V = rng.standard_normal((1, 2, L, d))
    exact = favor.softmax_attention(Q, K, V)
    errs = []
    for m in (16, 256, 4096, 16384):
        e = [np.abs(favor.favor_attention(Q, K, V, favor.make_features(s, m, d)) - exact).max()
             for s in range(20)]
        errs.append(float(np.mean(e)))
    assert all(a > b for a, b in zip(errs, errs[1:])), errs
    assert errs[-1] <= 1e-2, errs


def test_error_metrics():
    ref = np.array([1.0, -2.0, 0.0, 1.0])
    got = np.array([1.5, -2.0, 0.25, 1.0])
    ma, mr = favor.error_metrics(got, ref)
    assert ma == 0.5 and mr == pytest.approx(0.75 / 4.0)


# ---- incremental decoding ("Fast Transformer Decoding: One Write-Head is All You Need") ----
def test_decode_equals_causal_quadratic_form():
    # brute force: step t attends to keys 0..t with the explicit weights phi(q_t')^T phi(k_s')
    Q, K, V = _inputs(1, 4, 2, 9, 16, scale=0.5, seed=21)
    W = favor.make_features(4, 32, 16)
    got = favor.decode_outputs(Q, K, V, W)
    G = 2
    for h in range(4):
        phiq, _ = favor.query_features(Q[0, h], W, stabilise=False)
        phik, _ = favor.key_features(K[0, h // G], W, stabilise=False)
        A = np.tril(phiq @ phik.T)  # causal: key s <= query t
        want = (A @ V[0, h // G]) / A.sum(axis=1, keepdims=True)
        np.testing.assert_allclose(got[0, h], want, rtol=1e-12, atol=1e-12)


def test_decode_last_step_equals_bidirectional_attention():
    # after the last token the state holds every key: the bidirectional estimate for that query
    Q, K, V = _inputs(2, 2, 1, 12, 16, scale=0.5, seed=22)
    W = favor.make_features(5, 48, 16)
    got = favor.decode_outputs(Q, K, V, W)[:, :, -1]
    want = favor.favor_attention(Q, K, V, W)[:, :, -1]
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_decode_first_step_returns_the_first_value():
    # one key: every weight is on it, so the output is v_0 whatever the query
    Q, K, V = _inputs(1, 3, 1, 4, 16, scale=2.0, seed=23)
    W = favor.make_features(6, 32, 16)
    got = favor.decode_outputs(Q, K, V, W)
    for h in range(3):
        np.testing.assert_allclose(got[0, h, 0], V[0, 0, 0], rtol=1e-12, atol=1e-12)


# ---- generalised kernelizable attention with f = ReLU --------------------------------
# "Rethinking Attention with Performers", Abstract and RQ5: the same linear-time scheme
# for kernels other than softmax.  Pinned to the explicit L x L form, to the closed-form
# order-1 arc-cosine kernel the random features estimate, and to invariants of the map.
def test_relu_linear_order_equals_quadratic_form():
    Q, K, V = _inputs(1, 4, 2, 40, 16, seed=21)
    W = favor.make_features(5, 48, 16)
    G = 2
    want = np.empty_like(Q)
    for h in range(4):
        pq = favor.relu_features(Q[0, h], W)
        pk = favor.relu_features(K[0, h // G], W)
        A = pq @ pk.T
        want[0, h] = (A @ V[0, h // G]) / A.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(favor.relu_attention(Q, K, V, W), want, rtol=1e-11, atol=1e-12)


def test_relu_features_estimate_the_arccos_kernel():
    # E_w[relu(w.x) relu(w.y)] for w ~ N(0, I): the order-1 arc-cosine kernel; checked by
    # Monte Carlo over many iid draws, with the standard error as the yardstick
    d = 8
    rng = np.random.default_rng(22)
    x = rng.standard_normal(d)
    y = rng.standard_normal(d)
    W = favor.make_features(23, 200_000, d, orthogonal=False)
    prods = np.maximum(W @ x, 0) * np.maximum(W @ y, 0)
    nx, ny = np.linalg.norm(x), np.linalg.norm(y)
    t = math.acos(float(x @ y) / (nx * ny))
    closed = nx * ny * (math.sin(t) + (math.pi - t) * math.cos(t)) / (2 * math.pi)
    se = prods.std(ddof=1) / math.sqrt(prods.size)
    assert abs(prods.mean() - closed) < 4 * se, (prods.mean(), closed, se)
    assert se < 0.01 * closed


def test_relu_attention_converges_to_arccos_attention_as_m_grows():
    Q, K, V = _inputs(1, 1, 1, 24, 16, seed=24)
    want = favor.arccos1_attention(Q, K, V)
    errs = []
    for m in (64, 1024, 16384):
        W = favor.make_features(25, m, 16, orthogonal=False)
        errs.append(np.abs(favor.relu_attention(Q, K, V, W) - want).max())
    assert errs[0] > errs[1] > errs[2], errs
    assert errs[2] < 0.02, errs


def test_relu_attention_is_scale_free_and_convex():
    Q, K, V = _inputs(1, 2, 1, 30, 16, seed=26)
    W = favor.make_features(27, 64, 16)
    out = favor.relu_attention(Q, K, V, W)
    # positive homogeneity of relu: scaling queries or keys by a > 0 changes nothing
    np.testing.assert_allclose(favor.relu_attention(3.7 * Q, 0.25 * K, V, W), out, rtol=1e-11, atol=1e-12)
    lo, hi = V[0, 0].min(axis=0), V[0, 0].max(axis=0)
    assert np.all(out >= lo - 1e-12) and np.all(out <= hi + 1e-12)


def test_relu_attention_with_identical_keys_returns_the_mean_value():
    Q, K, V = _inputs(1, 1, 1, 20, 16, seed=28)
    K[:] = K[0, 0, 0]
    W = favor.make_features(29, 32, 16)
    out = favor.relu_attention(Q, K, V, W)
    np.testing.assert_allclose(out[0, 0], np.broadcast_to(V[0, 0].mean(axis=0), (20, 16)), rtol=1e-11, atol=1e-12)


# ---- trigonometric random features (the study's comparison point) ---------------------
def test_trig_feature_product_is_unbiased_for_softmax_kernel():
    d = 16
    rng = np.random.default_rng(42)
    q = rng.standard_normal(d) * 0.45
    k = rng.standard_normal(d) * 0.45
    est = np.empty(2000)
    for s in range(est.size):
        W = favor.make_features(20_000 + s, d, d, orthogonal=False)
        est[s] = float(favor.trig_features(q[None], W)[0] @ favor.trig_features(k[None], W)[0])
    target = math.exp(float(q @ k) / math.sqrt(d))
    se = est.std(ddof=1) / math.sqrt(est.size)
    assert abs(est.mean() - target) < 3.5 * se, (est.mean(), target, se)
    assert se < 0.05 * target


def test_trig_linear_order_equals_quadratic_form():
    Q, K, V = _inputs(1, 2, 1, 30, 16, scale=0.6, seed=43)
    W = favor.make_features(44, 24, 16)
    want = np.empty_like(Q)
    for h in range(2):
        A = favor.trig_features(Q[0, h], W) @ favor.trig_features(K[0, 0], W).T
        want[0, h] = (A @ V[0, 0]) / A.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(favor.trig_attention(Q, K, V, W), want, rtol=1e-9, atol=1e-10)


def test_trig_features_reproduce_the_gaussian_kernel_identity():
    # for one frequency row w: phi(x)^T phi(y) r = exp(|x'|^2/2 + |y'|^2/2) cos(w.(x' - y')), by the
    # angle-difference identity, whatever w is
    rng = np.random.default_rng(45)
    x, y = rng.standard_normal(8), rng.standard_normal(8)
    W = rng.standard_normal((1, 8))
    xs, ys = x * 8 ** -0.25, y * 8 ** -0.25
    want = math.exp(0.5 * (xs @ xs + ys @ ys)) * math.cos(float(W[0] @ (xs - ys)))
    got = float(favor.trig_features(x[None], W)[0] @ favor.trig_features(y[None], W)[0])
    assert abs(got - want) < 1e-12 * abs(want) + 1e-15
