"""GPU parity of Linformer projected attention (favor_linformer) against the fp64 oracle.

Linformer notes page, "4 Model": out = softmax(Q (E K)^T / sqrt(d)) (F V).  The same seeded
fp32 E and F go to both sides.  Tolerances as for FAVOR+: bf16 max-abs 2e-2 and mean-rel 5e-3,
fp32 1e-4 on both.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import linear_approximate_softmax_b200 as fv  # noqa: E402
from linear_approximate_softmax_b200 import workloads as wl  # noqa: E402
from oracle import favor as ofv  # noqa: E402
from oracle import linformer as olf  # noqa: E402

TOL = {torch.bfloat16: (2e-2, 5e-3), torch.float32: (1e-4, 1e-4)}


def f64(t):
    return t.float().numpy().astype(np.float64)


def run_linformer(Q, K, V, kp, seed=5, what="", report=None):
    L = Q.shape[2]
    E = olf.projection(seed, kp, L).astype(np.float32)
    F = olf.projection(seed + 1, kp, L).astype(np.float32)
    got = fv.favor_linformer(Q.cuda(), K.cuda(), V.cuda(), torch.from_numpy(E).cuda(), torch.from_numpy(F).cuda())
    fv.favor_device_check()
    got = f64(got.cpu())
    ref = olf.linformer_attention(f64(Q), f64(K), f64(V), E.astype(np.float64), F.astype(np.float64))
    ma, mr = ofv.error_metrics(got, ref)
    tol_abs, tol_rel = TOL[Q.dtype]
    assert np.all(np.isfinite(got)), what
    assert ma <= tol_abs and mr <= tol_rel, f"{what}: max-abs {ma:.3g} (<= {tol_abs}), mean-rel {mr:.3g} (<= {tol_rel})"
    if report is not None:
        report(f"linformer {what}: max-abs {ma:.3g} (limit {tol_abs}), mean-rel {mr:.3g} (limit {tol_rel})")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("d,kp", [(64, 64), (64, 256), (128, 128), (64, 512), (128, 256), (64, 80)])
def test_linformer_shapes(dtype, d, kp):
    Q, K, V = wl.random_inputs(1, 2, 2, 600, d, dtype, seed=d + kp)
    run_linformer(Q, K, V, kp, what=f"d={d} kp={kp} {dtype}")


@pytest.mark.parametrize("L", [1, 33, 300, 3001])
def test_linformer_ragged_lengths(L):
    Q, K, V = wl.random_inputs(1, 2, 1, L, 64, torch.bfloat16, seed=L + 9)
    run_linformer(Q, K, V, 64, what=f"L={L}")


@pytest.mark.parametrize("H,Hkv", [(6, 2), (8, 1)])
def test_linformer_grouped_heads(H, Hkv):
    Q, K, V = wl.random_inputs(2, H, Hkv, 400, 64, torch.bfloat16, seed=7 * H + Hkv)
    run_linformer(Q, K, V, 128, what=f"H={H} Hkv={Hkv}")


def test_linformer_identity_projection_is_softmax_attention():
    # k = L with E = F = I: exact softmax attention (the oracle's softmax_attention, itself pinned to SDPA)
    Q, K, V = wl.random_inputs(1, 2, 1, 128, 64, torch.float32, seed=11)
    I = torch.eye(128)
    got = f64(fv.favor_linformer(Q.cuda(), K.cuda(), V.cuda(), I.cuda(), I.cuda()).cpu())
    ref = ofv.softmax_attention(f64(Q), f64(K), f64(V))
    ma, mr = ofv.error_metrics(got, ref)
    assert ma <= 1e-4 and mr <= 1e-4, (ma, mr)


def test_linformer_full_size_headline_shape_every_element(parity_report):
    w = wl.WORKLOADS["bf16_L16384_heavykeys"]
    Q, K, V = wl.make_inputs(w)
    run_linformer(Q, K, V, 256, what=f"{w.name} kp=256 full size", report=parity_report)
