"""Plain fp64 CPU restatement of FAVOR+ attention (the oracle).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  It shares no code with ``linear_approximate_softmax_b200/``; the two
meet only through the seeded inputs that the tests hand to both.

What it computes follows "Rethinking Attention with Performers" (review page):
the Abstract and section 제안 방법 (proposed method) say that FAVOR+ estimates
the softmax attention kernel with *positive* *orthogonal* random features, in
linear time and space, and that the estimate is unbiased; section 주요 결과
(main results) says orthogonal and positive features lower the mean squared
error.  The pages do not print the formulas; the reading taken here is the
plainest one that those statements support:

* x' = d**-0.25 * x for queries and keys, so that exp(q'.k') = exp(q.k/sqrt(d))
  is the softmax kernel at the usual temperature;
* phi(x') = exp(W x' - |x'|^2 / 2) / sqrt(m) with W an m x d matrix of random
  rows, so that E_w[phi(q')^T phi(k')] * m / m = exp(q'.k') (unbiasedness);
* W: rows drawn N(0, I_d), orthogonalised in blocks of d rows (Gram-Schmidt,
  fp64, each projection applied twice), then each row rescaled to the length
  of an independent N(0, I_d) draw (a chi(d) norm), so every row is still
  marginally N(0, I_d); ``orthogonal=False`` keeps the raw iid rows;
* out = phi(Q') (phi(K')^T [V | 1]) / last column, never forming L x L
  (Abstract: linear space and time);
* stabilisers: one constant per (batch, kv-head) subtracted from every key
  exponent and one per query row subtracted from that row's exponents.  Both
  cancel exactly in the ratio; they only keep exp() in range.
* multi-query layout ("Fast Transformer Decoding: One Write-Head is All You
  Need", 提出的方法 / proposed method): H query heads share Hkv key/value heads;
  query head h reads kv head h // (H / Hkv).

Everything is fp64 and written step by step; numpy's matmul, exp and max are
the only library primitives used.
"""
import math

import numpy as np

from . import philox

TAG_DIRECTIONS = 0   # stream of the Gaussian rows that are orthogonalised
TAG_NORMS = 1        # stream of the Gaussian vectors whose lengths become row norms


# --------------------------------------------------------------------------
# Random features W  ("Rethinking Attention with Performers", Abstract and
# 제안 방법: positive orthogonal random features)
# --------------------------------------------------------------------------
def gram_schmidt_rows(G):
    """Orthonormalise the rows of a square fp64 matrix, first row first.

    Row i loses its components along rows 0..i-1 (all coefficients taken from
    the same vector, then subtracted), done twice so the result stays
    orthogonal to rounding level, and is then scaled to unit length.
    """
    G = np.asarray(G, dtype=np.float64)
    n = G.shape[0]
    Qm = np.zeros_like(G)
    for i in range(n):
        v = G[i].copy()
        for _ in range(2):
            if i:
                coef = Qm[:i] @ v
                v = v - Qm[:i].T @ coef
        Qm[i] = v / math.sqrt(float(v @ v))
    return Qm


def make_features(seed, m, d, orthogonal=True):
    """The m x d random-feature matrix W in fp64 (before storage rounding).

    orthogonal: ceil(m/d) independent d x d Gaussian blocks, each
    orthonormalised by rows; the first m rows of the stacked blocks are kept
    and row r is scaled to |h_r| for an independent h_r ~ N(0, I_d).
    iid: the first m rows of the same Gaussian stream, unchanged.
    """
    nblk = (m + d - 1) // d
    g = philox.normals(seed, TAG_DIRECTIONS, nblk * d * d).reshape(nblk, d, d)
    if not orthogonal:
        return g.reshape(nblk * d, d)[:m].copy()
    dirs = np.concatenate([gram_schmidt_rows(g[b]) for b in range(nblk)], axis=0)[:m]
    h = philox.normals(seed, TAG_NORMS, m * d).reshape(m, d)
    norms = np.sqrt(np.sum(h * h, axis=1))
    return dirs * norms[:, None]


def make_features_f32(seed, m, d, orthogonal=True):
    """W as the library stores it: the fp64 matrix rounded to fp32."""
    return make_features(seed, m, d, orthogonal).astype(np.float32)


# --------------------------------------------------------------------------
# Feature map and the linear-time estimate (Abstract: linear space and time)
# --------------------------------------------------------------------------
def scale_inputs(X):
    """x' = d**-1/4 x, so that q'.k' = q.k / sqrt(d)."""
    X = np.asarray(X, dtype=np.float64)
    return X * X.shape[-1] ** -0.25


def exponents(Xs, W):
    """Rows of W x' - |x'|^2/2 for every scaled row x' of Xs ([n, m])."""
    W = np.asarray(W, dtype=np.float64)
    return Xs @ W.T - 0.5 * np.sum(Xs * Xs, axis=1, keepdims=True)


def key_features(K, W, stabilise=True):
    """phi(K') for one kv head, and the key stabiliser that was subtracted.

    The key stabiliser is one constant, the largest exponent of the head, so
    that every key feature is at most 1/sqrt(m).
    """
    m = W.shape[0]
    u = exponents(scale_inputs(K), W)
    c = float(u.max()) if stabilise else 0.0
    return np.exp(u - c) / math.sqrt(m), c


def query_features(Q, W, stabilise=True):
    """phi(Q') for one query head; each row has its own stabiliser (its max)."""
    m = W.shape[0]
    u = exponents(scale_inputs(Q), W)
    c = u.max(axis=1, keepdims=True) if stabilise else np.zeros((u.shape[0], 1))
    return np.exp(u - c) / math.sqrt(m), c


def key_state(K, V, W, stabilise=True):
    """S = phi(K')^T [V | 1], an m x (d+1) matrix, with its key stabiliser."""
    phik, c = key_features(K, W, stabilise)
    V = np.asarray(V, dtype=np.float64)
    V1 = np.concatenate([V, np.ones((V.shape[0], 1))], axis=1)
    return phik.T @ V1, c


def query_output(Q, W, S, stabilise=True):
    """out_i = (phi(q_i')^T S[:, :d]) / (phi(q_i')^T S[:, d])."""
    phiq, _ = query_features(Q, W, stabilise)
    nz = phiq @ S
    d = S.shape[1] - 1
    return nz[:, :d] / nz[:, d:d + 1]


def favor_attention(Q, K, V, W, stabilise=True):
    """FAVOR+ bidirectional attention, fp64.

    Q: [B, H, L, d]; K, V: [B, Hkv, Lk, d]; W: [m, d].  H % Hkv == 0 and
    query head h reads kv head h // (H // Hkv).  Returns [B, H, L, d] fp64.
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    B, H, L, d = Q.shape
    Hkv = K.shape[1]
    assert H % Hkv == 0
    G = H // Hkv
    out = np.empty((B, H, L, d), dtype=np.float64)
    for b in range(B):
        for g in range(Hkv):
            S, _ = key_state(K[b, g], V[b, g], W, stabilise)
            for h in range(g * G, (g + 1) * G):
                out[b, h] = query_output(Q[b, h], W, S, stabilise)
    return out


def favor_quadratic(Q, K, V, W):
    """The same estimate with the L x L matrix formed: D^-1 (phi(Q') phi(K')^T) V.

    Only for tiny L; it checks that the linear-time order of products in
    ``favor_attention`` changes nothing but rounding.
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    B, H, L, d = Q.shape
    G = H // K.shape[1]
    out = np.empty((B, H, L, d), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            phiq, _ = query_features(Q[b, h], W)
            phik, _ = key_features(K[b, h // G], W)
            A = phiq @ phik.T
            out[b, h] = (A @ V[b, h // G]) / A.sum(axis=1, keepdims=True)
    return out


def softmax_attention(Q, K, V):
    """Exact softmax(Q K^T / sqrt(d)) V in fp64, the quantity FAVOR+ estimates."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    B, H, L, d = Q.shape
    G = H // K.shape[1]
    out = np.empty((B, H, L, d), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            s = Q[b, h] @ K[b, h // G].T / math.sqrt(d)
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            out[b, h] = (p @ V[b, h // G]) / p.sum(axis=1, keepdims=True)
    return out


# --------------------------------------------------------------------------
# Incremental decoding against the FAVOR+ state ("Fast Transformer Decoding:
# One Write-Head is All You Need", 研究动机与目标 / motivation and 提出的方法 /
# proposed method: one token at a time, with H query heads sharing one K/V
# head; here the cached K/V of each head is replaced by its fixed-size state)
# --------------------------------------------------------------------------
def decode_outputs(Q, K, V, W):
    """Outputs of T decoding steps, fp64.

    Q: [B, H, T, d], K, V: [B, Hkv, T, d].  Step t appends key/value t to each
    kv head's state and answers query t against it: the state after t + 1
    tokens is S_t = phi(K'[:t+1])^T [V[:t+1] | 1] (key_state of the first t + 1
    keys, one stabiliser for the whole head, which cancels), and
    out[:, :, t] = query_output(Q[:, :, t], W, S_t).  Returns [B, H, T, d].
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    B, H, T, d = Q.shape
    Hkv = K.shape[1]
    G = H // Hkv
    out = np.empty((B, H, T, d), dtype=np.float64)
    for b in range(B):
        for g in range(Hkv):
            # phi(K') of every key with one stabiliser for the head, then the running sum over
            # tokens: S_t is the sum of the first t + 1 rank-one terms phi(k_s)[v_s | 1]^T
            phik, _ = key_features(K[b, g], W)
            V1 = np.concatenate([V[b, g], np.ones((T, 1))], axis=1)
            S = np.zeros((W.shape[0], d + 1))
            for t in range(T):
                S = S + np.outer(phik[t], V1[t])
                for h in range(g * G, (g + 1) * G):
                    out[b, h, t] = query_output(Q[b, h, t:t + 1], W, S)[0]
    return out


# --------------------------------------------------------------------------
# Trigonometric random features, the comparison point of the feature-map
# study ("Rethinking Attention with Performers", 제안 방법 / proposed method:
# positive features instead of the usual sin/cos ones; 주요 결과 / main results:
# positive and orthogonal features lower the error).  With r rows of W,
# phi(x') = exp(|x'|^2/2) / sqrt(r) [sin(W x'), cos(W x')] (2r features):
# sin a sin b + cos a cos b = cos(a - b) and E_w cos(w.z) = exp(-|z|^2/2) for
# w ~ N(0, I), so E[phi(q')^T phi(k')] = exp(q'.k').  Its weights can be
# negative, so no stabiliser applies and the ratio can leave V's hull.
# --------------------------------------------------------------------------
def trig_features(X, W):
    """exp(|x'|^2/2) / sqrt(r) [sin(W x'), cos(W x')] for every scaled row x' of X ([n, 2r])."""
    W = np.asarray(W, dtype=np.float64)
    Xs = scale_inputs(X)
    u = Xs @ W.T
    amp = np.exp(0.5 * np.sum(Xs * Xs, axis=1, keepdims=True)) / math.sqrt(W.shape[0])
    return amp * np.concatenate([np.sin(u), np.cos(u)], axis=1)


def trig_attention(Q, K, V, W):
    """The linear-time estimate with trigonometric features, per kv head, fp64 (shapes as favor_attention)."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    B, H, L, d = Q.shape
    G = H // K.shape[1]
    out = np.empty((B, H, L, d), dtype=np.float64)
    for b in range(B):
        for g in range(K.shape[1]):
            V1 = np.concatenate([V[b, g], np.ones((V.shape[2], 1))], axis=1)
            S = trig_features(K[b, g], W).T @ V1
            for h in range(g * G, (g + 1) * G):
                nz = trig_features(Q[b, h], W) @ S
                out[b, h] = nz[:, :d] / nz[:, d:d + 1]
    return out


# --------------------------------------------------------------------------
# Generalised kernelizable attention, f = ReLU ("Rethinking Attention with
# Performers", Abstract: the method also approximates kernelizable attention
# other than softmax; 연구 질문 / research questions, RQ5).  The pages name no
# f; the reading taken here is the plainest one: phi(x) = ReLU(W x') / sqrt(m)
# with the same x' = d**-0.25 x and the same W, and the same linear-time order
# of products.  ReLU is positively homogeneous, so the input scaling and the
# 1/sqrt(m) factor cancel in the ratio; no stabiliser is needed (phi >= 0 and
# bounded by |W x'|).
# --------------------------------------------------------------------------
def relu_features(X, W):
    """phi(x') = max(W x', 0) / sqrt(m) for every scaled row x' of X ([n, m])."""
    W = np.asarray(W, dtype=np.float64)
    return np.maximum(scale_inputs(X) @ W.T, 0.0) / math.sqrt(W.shape[0])


def relu_attention(Q, K, V, W):
    """out = phi(Q') (phi(K')^T [V | 1]) / last column, per kv head, fp64.

    Shapes as in ``favor_attention``.  A query whose features all vanish
    against every key (denominator 0) has no defined output; the division
    is left to produce it (inf or nan).
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    B, H, L, d = Q.shape
    Hkv = K.shape[1]
    assert H % Hkv == 0
    G = H // Hkv
    out = np.empty((B, H, L, d), dtype=np.float64)
    for b in range(B):
        for g in range(Hkv):
            phik = relu_features(K[b, g], W)
            V1 = np.concatenate([V[b, g], np.ones((V.shape[2], 1))], axis=1)
            S = phik.T @ V1
            for h in range(g * G, (g + 1) * G):
                nz = relu_features(Q[b, h], W) @ S
                out[b, h] = nz[:, :d] / nz[:, d:d + 1]
    return out


def arccos1_attention(Q, K, V):
    """The attention that relu_attention estimates as m grows with iid N(0, I) rows of W.

    E_w[max(w.x, 0) max(w.y, 0)] = |x| |y| (sin t + (pi - t) cos t) / (2 pi), t the
    angle between x and y (the order-1 arc-cosine kernel), so the weights are
    that kernel of the scaled rows, normalised over the keys; computed with the
    L x L matrix formed.
    """
    Q = scale_inputs(Q)
    K = scale_inputs(K)
    V = np.asarray(V, dtype=np.float64)
    B, H, L, d = Q.shape
    G = H // K.shape[1]
    out = np.empty((B, H, L, d), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            q, k = Q[b, h], K[b, h // G]
            nq = np.sqrt(np.sum(q * q, axis=1))[:, None]
            nk = np.sqrt(np.sum(k * k, axis=1))[None, :]
            cos = np.clip((q @ k.T) / (nq * nk), -1.0, 1.0)
            t = np.arccos(cos)
            A = nq * nk * (np.sin(t) + (math.pi - t) * cos) / (2 * math.pi)
            out[b, h] = (A @ V[b, h // G]) / A.sum(axis=1, keepdims=True)
    return out


# --------------------------------------------------------------------------
# Error metrics used by every parity test
# --------------------------------------------------------------------------
def error_metrics(got, ref):
    """max |got - ref| and sum |got - ref| / sum |ref| (the mean relative error)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    diff = np.abs(got - ref)
    return float(diff.max()) if diff.size else 0.0, float(diff.sum() / max(np.abs(ref).sum(), 1e-300))
