"""GPU parity of the generalised kernelizable attention with f = ReLU against the fp64 oracle.

"Rethinking Attention with Performers" (Abstract; RQ5): the same linear-time scheme for
kernels other than softmax, here phi(x) = ReLU(W x') / sqrt(m).  Tolerances as for
FAVOR+: bf16 inputs max-abs 2e-2 and mean-rel 5e-3, fp32 inputs 1e-4 on both.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import linear_approximate_softmax_b200 as fv  # noqa: E402
from linear_approximate_softmax_b200 import workloads as wl  # noqa: E402
from oracle import favor as ofv  # noqa: E402

TOL = {torch.bfloat16: (2e-2, 5e-3), torch.float32: (1e-4, 1e-4)}


def f64(t):
    return t.float().numpy().astype(np.float64)


def run_relu(Q, K, V, m, seed=1, orthogonal=True, what="", report=None):
    d = Q.shape[-1]
    W = fv.favor_make_features(seed, m, d, orthogonal)
    got = fv.favor_attention_relu(Q.cuda(), K.cuda(), V.cuda(), W.cuda())
    fv.favor_device_check()
    got = f64(got.cpu())
    ref = ofv.relu_attention(f64(Q), f64(K), f64(V), ofv.make_features_f32(seed, m, d, orthogonal))
    ma, mr = ofv.error_metrics(got, ref)
    tol_abs, tol_rel = TOL[Q.dtype]
    assert np.all(np.isfinite(got)), what
    assert ma <= tol_abs and mr <= tol_rel, f"{what}: max-abs {ma:.3g} (<= {tol_abs}), mean-rel {mr:.3g} (<= {tol_rel})"
    lo = f64(V).min(axis=2, keepdims=True)
    hi = f64(V).max(axis=2, keepdims=True)
    G = Q.shape[1] // K.shape[1]
    lo, hi = np.repeat(lo, G, axis=1), np.repeat(hi, G, axis=1)
    tol = 1e-2 if Q.dtype == torch.bfloat16 else 1e-5
    assert np.all(got >= lo - tol) and np.all(got <= hi + tol), f"{what}: outside the convex hull of V"
    if report is not None:
        report(f"relu {what}: max-abs {ma:.3g} (limit {tol_abs}), mean-rel {mr:.3g} (limit {tol_rel})")
    return ma, mr


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("d,m", [(64, 64), (64, 256), (128, 128), (64, 512), (128, 256)])
def test_relu_shapes(dtype, d, m):
    Q, K, V = wl.random_inputs(1, 2, 2, 700, d, dtype, seed=d + m)
    run_relu(Q, K, V, m, what=f"d={d} m={m} {dtype}")


@pytest.mark.parametrize("L", [1, 31, 129, 1000])
def test_relu_ragged_lengths(L):
    Q, K, V = wl.random_inputs(1, 2, 1, L, 64, torch.bfloat16, seed=L + 5)
    run_relu(Q, K, V, 128, what=f"L={L}")


@pytest.mark.parametrize("H,Hkv", [(6, 2), (8, 1)])
def test_relu_grouped_heads(H, Hkv):
    Q, K, V = wl.random_inputs(2, H, Hkv, 300, 64, torch.bfloat16, seed=H + 3 * Hkv)
    run_relu(Q, K, V, 256, what=f"H={H} Hkv={Hkv}")


def test_relu_iid_features():
    Q, K, V = wl.random_inputs(1, 2, 2, 500, 64, torch.float32, seed=77)
    run_relu(Q, K, V, 256, orthogonal=False, what="iid W")


def test_relu_full_size_headline_shape_every_element(parity_report):
    # the headline shape (B4 H12 L16384 d64 m256, bf16, heavy-tailed key norms), every element
    w = wl.WORKLOADS["bf16_L16384_heavykeys"]
    Q, K, V = wl.make_inputs(w)
    run_relu(Q, K, V, w.m, w.w_seed, True, f"{w.name} full size", parity_report)


def test_relu_query_rows_scaled_by_powers_of_two():
    # phi(c q) = c phi(q) for c > 0, so each query row's output does not depend on its scale.  Rows
    # scaled by 2^-30 .. 2^30 (exact in bf16) drive the tensor-core query pass's integer row
    # stabiliser over its whole range, including raises after a row's first feature block.
    Q, K, V = wl.random_inputs(1, 4, 2, 600, 64, torch.bfloat16, seed=91)
    rng = np.random.default_rng(5)
    e = torch.from_numpy(rng.integers(-30, 31, size=(1, 4, 600, 1)).astype(np.float32))
    Qs = (Q.float() * torch.exp2(e)).to(torch.bfloat16)
    assert torch.equal(Qs.float(), Q.float() * torch.exp2(e))
    for m in (128, 256, 512):
        run_relu(Qs, K, V, m, what=f"rows scaled by 2^-30..2^30, m={m}")
        W = fv.favor_make_features(1, m, 64).cuda()
        a = fv.favor_attention_relu(Qs.cuda(), K.cuda(), V.cuda(), W).float()
        b = fv.favor_attention_relu(Q.cuda(), K.cuda(), V.cuda(), W).float()
        fv.favor_device_check()
        assert (a - b).abs().max().item() <= 2e-2, m
