"""Plain fp64 CPU restatement of Linformer projected attention (oracle).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  It shares no code with ``linear_approximate_softmax_b200/``.

What it computes follows the Linformer notes page, section "4 Model": the keys
and values of each head are projected along the sequence by two matrices E and
F of k rows and n (here L) columns, and attention runs over the k projected
rows:  out = softmax(Q (E K)^T / sqrt(d)) (F V).  The pages use trained E and
F; the tests pass seeded Gaussian ones with entries N(0, 1/L), the plainest
stand-in: a random projection of the sequence whose rows, like an average over
the tokens, keep the scale of the rows of K and V (so outputs stay on V's scale
and the tolerances of the other workloads apply as stated).  One E and one F serve every
head of a call (the page's shared-projection option); query heads that share a
key/value head (multi-query layout) share its projected rows.
"""
import math

import numpy as np


def projection(seed, k, L):
    """A seeded k x L matrix with N(0, 1/L) entries (numpy's generator; an input, not part of the method)."""
    rng = np.random.default_rng(seed)
    return rng.standard_normal((k, L)) / math.sqrt(L)


def linformer_attention(Q, K, V, E, F):
    """softmax(Q (E K)^T / sqrt(d)) (F V) per head, fp64.

    Q: [B, H, L, d]; K, V: [B, Hkv, L, d]; E, F: [k, L].  Query head h reads
    kv head h // (H / Hkv).  Returns [B, H, L, d].
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    E = np.asarray(E, dtype=np.float64)
    F = np.asarray(F, dtype=np.float64)
    B, H, L, d = Q.shape
    Hkv = K.shape[1]
    assert H % Hkv == 0 and E.shape[1] == L and F.shape[1] == L
    G = H // Hkv
    out = np.empty((B, H, L, d), dtype=np.float64)
    for b in range(B):
        for g in range(Hkv):
            Kp = E @ K[b, g]  # [k, d]: the projected keys
            Vp = F @ V[b, g]  # [k, d]: the projected values
            for h in range(g * G, (g + 1) * G):
                s = Q[b, h] @ Kp.T / math.sqrt(d)
                s = s - s.max(axis=1, keepdims=True)
                p = np.exp(s)
                out[b, h] = (p @ Vp) / p.sum(axis=1, keepdims=True)
    return out
