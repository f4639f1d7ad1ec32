"""Write oracle_small.json from the oracle alone (run from the repo root)."""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import favor  # noqa: E402


def case():
    rng = np.random.default_rng(2024)
    Q = rng.standard_normal((1, 2, 5, 16)) * 0.5
    K = rng.standard_normal((1, 1, 5, 16)) * 0.5
    V = rng.standard_normal((1, 1, 5, 16))
    return Q, K, V


if __name__ == "__main__":
    Q, K, V = case()
    W = favor.make_features(3, 32, 16)
    out = favor.favor_attention(Q, K, V, W)
    doc = {
        "what": "oracle FAVOR+ output, B=1 H=2 Hkv=1 L=5 d=16 m=32, W seed 3 orthogonal; inputs from numpy default_rng(2024)",
        "W_first_row": W[0].tolist(),
        "out": out.reshape(-1).tolist(),
    }
    with open(os.path.join(HERE, "oracle_small.json"), "w") as f:
        json.dump(doc, f, indent=1)
