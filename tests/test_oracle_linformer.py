"""Pins for the oracle's Linformer projected attention (Linformer notes page, "4 Model").

Each check ties the projected attention to something fixed outside it: torch's
scaled-dot-product attention when the projections are the identity or a
permutation, linearity in the values, and the convex hull of the projected values.
"""
import math

import numpy as np
import torch

from oracle import linformer


def _inputs(B, H, Hkv, L, d, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, H, L, d)), rng.standard_normal((B, Hkv, L, d)),
            rng.standard_normal((B, Hkv, L, d)))


def _sdpa(Q, K, V, G):
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q), torch.from_numpy(K).repeat_interleave(G, dim=1),
        torch.from_numpy(V).repeat_interleave(G, dim=1)).numpy()


def test_identity_projections_give_softmax_attention():
    Q, K, V = _inputs(2, 4, 2, 37, 16, seed=31)
    I = np.eye(37)
    np.testing.assert_allclose(linformer.linformer_attention(Q, K, V, I, I), _sdpa(Q, K, V, 2), rtol=1e-10, atol=1e-12)


def test_permutation_projections_give_softmax_attention():
    # attention does not depend on the order of the key/value pairs when both move together
    Q, K, V = _inputs(1, 2, 1, 29, 8, seed=32)
    P = np.eye(29)[np.random.default_rng(33).permutation(29)]
    np.testing.assert_allclose(linformer.linformer_attention(Q, K, V, P, P), _sdpa(Q, K, V, 2), rtol=1e-10, atol=1e-12)


def test_projected_attention_matches_sdpa_on_the_projected_rows():
    # with k < L the result is attention over the k rows E K and F V, formed here by hand
    Q, K, V = _inputs(1, 3, 1, 50, 16, seed=34)
    E, F = linformer.projection(35, 12, 50), linformer.projection(36, 12, 50)
    Kp = np.einsum("kl,bhld->bhkd", E, K)
    Vp = np.einsum("kl,bhld->bhkd", F, V)
    np.testing.assert_allclose(linformer.linformer_attention(Q, K, V, E, F), _sdpa(Q, Kp, Vp, 3), rtol=1e-10, atol=1e-12)


def test_linear_in_the_values_and_inside_the_projected_hull():
    Q, K, V = _inputs(1, 2, 2, 40, 16, seed=37)
    V2 = np.random.default_rng(38).standard_normal(V.shape)
    E, F = linformer.projection(39, 16, 40), linformer.projection(40, 16, 40)
    a = linformer.linformer_attention(Q, K, V, E, F)
    b = linformer.linformer_attention(Q, K, V2, E, F)
    np.testing.assert_allclose(linformer.linformer_attention(Q, K, V + 2.5 * V2, E, F), a + 2.5 * b, rtol=1e-10, atol=1e-11)
    Vp = np.einsum("kl,bhld->bhkd", F, V)
    assert np.all(a >= Vp.min(axis=2, keepdims=True) - 1e-12) and np.all(a <= Vp.max(axis=2, keepdims=True) + 1e-12)


def test_projection_entries_have_variance_one_over_L():
    E = linformer.projection(41, 64, 4096)
    assert abs(E.mean()) < 4 / math.sqrt(E.size) / math.sqrt(4096)
    assert abs(E.var() * 4096 - 1.0) < 0.02
