"""GPU parity of incremental decoding against the fp64 oracle.

"Fast Transformer Decoding: One Write-Head is All You Need" (研究动机与目标 /
motivation; 提出的方法 / proposed method): tokens arrive one at a time and
several query heads may share one key/value head; here each kv head's cache is
its FAVOR+ state.  The oracle's decode_outputs restates step t as the query
pass over the state of the first t + 1 keys.  Tolerances as for the full
attention: bf16 max-abs <= 2e-2 and mean-rel <= 5e-3, fp32 1e-4.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import linear_approximate_softmax_b200 as fv  # noqa: E402
from linear_approximate_softmax_b200 import workloads as wl  # noqa: E402
from oracle import favor as ofv  # noqa: E402

TOL = {torch.bfloat16: (2e-2, 5e-3), torch.float32: (1e-4, 1e-4)}


def run_decode(Q, K, V, W):
    """All T steps on the GPU from an empty state; returns [B, H, T, d] on the host."""
    B, H, T, d = Q.shape
    Hkv, m = K.shape[1], W.shape[0]
    Qd, Kd, Vd, Wd = Q.cuda(), K.cuda(), V.cuda(), W.cuda()
    state = torch.empty(fv.favor_decode_state_bytes(B, Hkv, d, m), dtype=torch.uint8, device="cuda")
    fv.favor_decode_init(state, B, Hkv, d, m)
    outs = torch.empty(T, B, H, d, dtype=Q.dtype, device="cuda")
    for t in range(T):
        fv.favor_decode_step(Qd[:, :, t].contiguous(), Kd[:, :, t].contiguous(), Vd[:, :, t].contiguous(), Wd,
                             state, outs[t])
    fv.favor_device_check()
    return outs.permute(1, 2, 0, 3).cpu()


@pytest.mark.parametrize("dtype,B,H,Hkv,T,d,m", [
    (torch.bfloat16, 2, 4, 1, 1000, 128, 256),   # multi-query: four query heads share one kv head
    (torch.bfloat16, 1, 6, 2, 400, 64, 512),
    (torch.float32, 1, 2, 2, 300, 64, 128),
    (torch.bfloat16, 1, 64, 1, 120, 128, 512),   # the most query heads per kv head, the most features
    (torch.float32, 2, 17, 1, 150, 64, 16),      # an odd group of query heads, two features per CTA
    (torch.bfloat16, 3, 10, 2, 100, 128, 208),   # 26 features per CTA: not a power of two
])
def test_decode_matches_oracle(dtype, B, H, Hkv, T, d, m, parity_report):
    Q, K, V = wl.random_inputs(B, H, Hkv, T, d, dtype, seed=T + d)
    W = fv.favor_make_features(1, m, d)
    got = run_decode(Q, K, V, W).float().numpy().astype(np.float64)
    ref = ofv.decode_outputs(*[t.float().numpy().astype(np.float64) for t in (Q, K, V)], ofv.make_features_f32(1, m, d))
    max_abs, mean_rel = ofv.error_metrics(got, ref)
    tol_abs, tol_rel = TOL[dtype]
    parity_report(f"decode {str(dtype).split('.')[-1]} B{B} H{H} Hkv{Hkv} T{T} d{d} m{m}: max-abs {max_abs:.3g} "
                  f"(limit {tol_abs:g}), mean-rel {mean_rel:.3g} (limit {tol_rel:g})")
    assert np.all(np.isfinite(got))
    assert max_abs <= tol_abs and mean_rel <= tol_rel, (max_abs, mean_rel)


def test_decode_state_equals_key_pass_state():
    # after T steps the decode state, brought to one stabiliser, equals the key pass's reduced state
    B, H, Hkv, T, d, m = 1, 2, 2, 500, 64, 128
    Q, K, V = wl.random_inputs(B, H, Hkv, T, d, torch.float32, seed=3)
    W = fv.favor_make_features(2, m, d)
    Kd, Vd, Wd = K.cuda(), V.cuda(), W.cuda()
    state = torch.empty(fv.favor_decode_state_bytes(B, Hkv, d, m), dtype=torch.uint8, device="cuda")
    fv.favor_decode_init(state, B, Hkv, d, m)
    for t in range(T):
        fv.favor_decode_step(Q[:, :, t].contiguous().cuda(), Kd[:, :, t].contiguous(), Vd[:, :, t].contiguous(), Wd,
                             state, torch.empty(B, H, d, device="cuda"))
    fv.favor_device_check()
    # per kv head: S [m][d + 1], then c [m]
    st = state.view(torch.float32).view(B * Hkv, m * (d + 2)).double().cpu().numpy()
    S, c = st[:, :m * (d + 1)].reshape(B * Hkv, m, d + 1), st[:, m * (d + 1):]
    Wo = ofv.make_features_f32(2, m, d)
    for hk in range(B * Hkv):
        So, _ = ofv.key_state(K[0, hk].double().numpy(), V[0, hk].double().numpy(), Wo)
        Sg = S[hk] * np.exp2(c[hk] - c[hk].max())[:, None]  # the state relative to one constant
        gn, on = Sg / Sg[:, d].sum(), So / So[:, d].sum()
        assert np.abs(gn - on).max() <= 1e-5 * np.abs(on).max()
