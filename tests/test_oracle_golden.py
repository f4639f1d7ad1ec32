"""The oracle reproduces its stored small-case output (a regression guard)."""
import json
import os

import numpy as np

from oracle import favor

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_matches_stored_small_case():
    import importlib.util
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(HERE, "golden", "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    doc = json.load(open(os.path.join(HERE, "golden", "oracle_small.json")))
    Q, K, V = mg.case()
    W = favor.make_features(3, 32, 16)
    np.testing.assert_allclose(W[0], doc["W_first_row"], rtol=1e-13)
    np.testing.assert_allclose(favor.favor_attention(Q, K, V, W).reshape(-1), doc["out"], rtol=1e-11)
