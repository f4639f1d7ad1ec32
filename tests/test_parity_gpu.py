"""GPU parity: the CUDA path against the fp64 oracle on identical seeded inputs.

Tolerances (fixed for this library): bf16 inputs with fp32 accumulation must
reach max |gpu - oracle| <= 2e-2 and sum|gpu - oracle| / sum|oracle| <= 5e-3;
fp32 inputs must reach 1e-4 on both.  The GPU gets W from the library's
favor_make_features, the oracle from its own generator (the two are checked
equal on the CPU in test_abi.py).
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


def gpu_attention(Q, K, V, W):
    out = fv.favor_attention(Q.cuda(), K.cuda(), V.cuda(), W.cuda())
    fv.favor_device_check()  # synchronises; raises if a kernel gave up waiting
    return out.cpu()


def assert_close(got, ref, dtype, what=""):
    ma, mr = ofv.error_metrics(f64(got) if torch.is_tensor(got) else got, ref)
    tol_abs, tol_rel = TOL[dtype]
    assert np.all(np.isfinite(f64(got) if torch.is_tensor(got) else got)), what
    assert ma <= tol_abs and mr <= tol_rel, f"{what}: max-abs {ma:.3g} (<= {tol_abs}), mean-rel {mr:.3g} (<= {tol_rel})"
    return ma, mr


def run_case(Q, K, V, m, seed=1, orthogonal=True, what=""):
    d = Q.shape[-1]
    W = fv.favor_make_features(seed, m, d, orthogonal)
    got = gpu_attention(Q, K, V, W)
    ref = ofv.favor_attention(f64(Q), f64(K), f64(V), ofv.make_features_f32(seed, m, d, orthogonal))
    return assert_close(got, ref, Q.dtype, what)


# ---- the five workloads at sizes the oracle runs element-wise in seconds ----
SMALL = {
    "fp32_L256": dict(),
    "bf16_L4096": dict(B=2, H=2, Hkv=2, L=1000),
    "bf16_L16384_heavykeys": dict(B=1, H=3, Hkv=3, L=2000),
    "bf16_mqa_L8192_d128": dict(B=2, H=4, Hkv=1, L=700),
    "bf16_L131072_m512": dict(B=1, H=2, Hkv=2, L=3000),
}


@pytest.mark.parametrize("name", wl.WORKLOAD_ORDER)
def test_workload_small_elementwise(name):
    w = wl.WORKLOADS[name]
    Q, K, V = wl.make_inputs(w, **SMALL[name])
    for orth in w.orthogonal:
        run_case(Q, K, V, w.m, w.w_seed, orth, f"{name} orthogonal={orth}")


# ---- edge cases: ragged and tiny L, m not a multiple of 64, grouped heads ----
@pytest.mark.parametrize("L", [1, 2, 127, 128, 129, 1000])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_ragged_lengths(L, dtype):
    Q, K, V = wl.random_inputs(1, 2, 1, L, 64, dtype, seed=L)
    run_case(Q, K, V, 64, what=f"L={L}")


@pytest.mark.parametrize("m", [16, 48, 80, 128, 192, 512])
@pytest.mark.parametrize("d", [64, 128])
def test_feature_counts(m, d):
    Q, K, V = wl.random_inputs(1, 2, 2, 300, d, torch.bfloat16, seed=m + d)
    run_case(Q, K, V, m, what=f"m={m} d={d}")


@pytest.mark.parametrize("H,Hkv", [(6, 2), (8, 1), (4, 4)])
def test_grouped_heads(H, Hkv):
    Q, K, V = wl.random_inputs(2, H, Hkv, 257, 64, torch.bfloat16, seed=H * 10 + Hkv)
    run_case(Q, K, V, 128, what=f"H={H} Hkv={Hkv}")


def test_large_norm_inputs_stay_finite():
    # exponents far below zero: only the stabilisers keep exp() in range
    Q, K, V = wl.random_inputs(1, 1, 1, 500, 64, torch.float32, seed=3, scale=6.0)
    run_case(Q, K, V, 128, what="scale 6")


def test_growing_key_norms_force_rescaling():
    # key norms rise along the sequence, so later chunks raise the running stabiliser
    Q, K, V = wl.random_inputs(1, 1, 1, 4000, 64, torch.float32, seed=4)
    ramp = torch.linspace(0.2, 3.0, 4000).view(1, 1, 4000, 1)
    run_case(Q, (K * ramp).contiguous(), V, 128, what="ramp")


def test_key_stabiliser_raised_late_bf16():
    # the first key tiles have near-zero exponents; later keys sit on random feature rows,
    # so their exponents are ~|w|^2/2 and the chunk stabiliser must be raised (and S rescaled)
    d, m, L = 64, 256, 1500
    W = fv.favor_make_features(1, m, d)
    g = torch.Generator().manual_seed(7)
    K = 0.01 * torch.randn(1, 1, L, d, generator=g)
    rows = torch.randint(0, m, (L,), generator=g)
    late = torch.arange(L) >= 300
    K[0, 0, late] = W[rows[late]] * d ** 0.25 * 0.7
    Q = torch.randn(1, 2, L, d, generator=g) * 0.5
    V = torch.randn(1, 1, L, d, generator=g)
    run_case(Q.bfloat16(), K.bfloat16(), V.bfloat16(), m, what="late keys")


def test_query_stabiliser_raised_in_second_feature_block_bf16():
    # each query sits on a feature row of the second 128-feature block, so its row max there
    # exceeds the first block's and the running output must be rescaled
    d, m, L = 64, 256, 700
    W = fv.favor_make_features(1, m, d)
    g = torch.Generator().manual_seed(8)
    rows = torch.randint(128, m, (L,), generator=g)
    Q = (W[rows] * d ** 0.25 * 0.6).view(1, 1, L, d).repeat(1, 2, 1, 1)
    K = torch.randn(1, 1, L, d, generator=g)
    V = torch.randn(1, 1, L, d, generator=g)
    run_case(Q.bfloat16(), K.bfloat16(), V.bfloat16(), m, what="late queries")


def test_scaled_query_rows_take_the_unfolded_path():
    # A query row whose largest |q| reaches 2^15 overflows fp16 as a projection operand, so it is
    # scaled by 2^-k, and every row of its 32-row group adds e_f on the CUDA cores instead of
    # through the projection.  The ordinary rows of such groups must still match the oracle; the
    # huge rows (whose exponents no fp16 projection resolves) must stay finite and inside the
    # per-column range of V, since every FAVOR+ weight is positive.
    d, m, L = 64, 256, 300
    g = torch.Generator().manual_seed(9)
    Q = torch.randn(1, 2, L, d, generator=g) * 0.5
    huge = [5, 40, 77, 130, 261]  # rows in four different 32-row groups and two 128-row tiles
    for i in huge:
        u = torch.randn(d, generator=g)
        Q[0, :, i] = 65536.0 * u / u.abs().max()
    K = torch.randn(1, 1, L, d, generator=g)
    V = torch.randn(1, 1, L, d, generator=g)
    Qb, Kb, Vb = Q.bfloat16(), K.bfloat16(), V.bfloat16()
    W = fv.favor_make_features(1, m, d)
    got = f64(gpu_attention(Qb, Kb, Vb, W))
    assert np.all(np.isfinite(got))
    ref = ofv.favor_attention(f64(Qb), f64(Kb), f64(Vb), ofv.make_features_f32(1, m, d))
    normal = np.setdiff1d(np.arange(L), huge)
    assert_close(got[:, :, normal], ref[:, :, normal], torch.bfloat16, "rows beside scaled rows")
    v = f64(Vb)[0, 0]
    lo, hi = v.min(axis=0) - 1e-2, v.max(axis=0) + 1e-2
    assert np.all((got[0, :, huge] >= lo) & (got[0, :, huge] <= hi))


# ---- full sizes, in the launch configuration bench.py times ----------------
def _bench_path(Qd, Kd, Vd, Wd):
    """The three stage calls back to back with launch overlap on, as bench.py times them."""
    B, H, L, d = Qd.shape
    Hkv, m = Kd.shape[1], Wd.shape[0]
    before = fv.favor_set_launch_overlap(True)
    try:
        part = torch.empty(fv.favor_partials_bytes(B, Hkv, L, d, m), dtype=torch.uint8, device="cuda")
        state = torch.empty(fv.favor_state_bytes(B, Hkv, d, m), dtype=torch.uint8, device="cuda")
        out = torch.empty_like(Qd)
        fv.favor_key_pass(Kd, Vd, Wd, part)
        fv.favor_state_reduce(part, state, B, Hkv, L, d, m)
        fv.favor_query_pass(Qd, Wd, state, Hkv, out)
        fv.favor_device_check()
    finally:
        fv.favor_set_launch_overlap(before)
    return out


@pytest.mark.parametrize("name,orth", [(n, o) for n in wl.WORKLOAD_ORDER for o in wl.WORKLOADS[n].orthogonal])
def test_workload_full_size_every_element(name, orth, parity_report):
    # every output element of the full-size workload against the oracle, head by head; at these
    # sizes the persistent query pass walks tens of tiles per CTA across head boundaries
    w = wl.WORKLOADS[name]
    Q, K, V = wl.make_inputs(w)
    W = fv.favor_make_features(w.w_seed, w.m, w.d, orth)
    Qd, Kd, Vd, Wd = Q.cuda(), K.cuda(), V.cuda(), W.cuda()
    out = _bench_path(Qd, Kd, Vd, Wd)
    fused = fv.favor_attention(Qd, Kd, Vd, Wd)
    fv.favor_device_check()
    assert torch.equal(out, fused)  # the same kernels through the one-call entry point
    out = out.cpu()
    del Qd, Kd, Vd, fused
    Wo = ofv.make_features_f32(w.w_seed, w.m, w.d, orth)
    G = w.H // w.Hkv
    max_abs, sum_diff, sum_ref, hull = 0.0, 0.0, 0.0, 0.0
    for b in range(w.B):
        for g in range(w.Hkv):
            v = f64(V[b, g])
            S, _ = ofv.key_state(f64(K[b, g]), v, Wo)
            lo, hi = v.min(0), v.max(0)
            for h in range(g * G, (g + 1) * G):
                ref = ofv.query_output(f64(Q[b, h]), Wo, S)
                got = f64(out[b, h])
                assert np.all(np.isfinite(got)), (b, h)
                diff = np.abs(got - ref)
                max_abs = max(max_abs, float(diff.max()))
                sum_diff += float(diff.sum())
                sum_ref += float(np.abs(ref).sum())
                # every row is a convex combination of the value rows (all weights positive)
                hull = max(hull, float(np.max(lo - got)), float(np.max(got - hi)))
    mean_rel = sum_diff / sum_ref
    tol_abs, tol_rel = TOL[w.dtype]
    parity_report(f"{name} W={'orthogonal' if orth else 'iid'}: {out.numel()} elements, max-abs {max_abs:.3g} "
                  f"(limit {tol_abs:g}, margin {tol_abs - max_abs:.3g}), mean-rel {mean_rel:.3g} "
                  f"(limit {tol_rel:g}, margin {tol_rel - mean_rel:.3g}), convex-hull excess {max(hull, 0.0):.3g}")
    assert max_abs <= tol_abs and mean_rel <= tol_rel, (max_abs, mean_rel)
    assert hull <= tol_abs


# ---- API equivalences -------------------------------------------------------
def test_deterministic_bitwise():
    w = wl.WORKLOADS["bf16_L4096"]
    Q, K, V = [t.cuda() for t in wl.make_inputs(w, B=2, H=4, Hkv=4, L=4096)]
    W = fv.favor_make_features(1, w.m, w.d).cuda()
    a = fv.favor_attention(Q, K, V, W)
    b = fv.favor_attention(Q, K, V, W)
    fv.favor_device_check()
    assert torch.equal(a, b)


def test_alternating_shapes_reuse_pool_memory():
    # Fused calls of two shapes in turn (d = 64 and the multi-query d = 128): each call's scratch
    # comes back from the stream-ordered pool holding the other shape's partial state and state.
    # Every kernel must read only what its call wrote, with reads of a preceding kernel's output
    # that stay coherent while that kernel was still writing (programmatic launches): every
    # repetition equals the first, bit for bit, and is finite.
    a = [t.cuda() for t in wl.random_inputs(1, 3, 3, 2000, 64, torch.bfloat16, seed=41)]
    b = [t.cuda() for t in wl.random_inputs(2, 4, 1, 700, 128, torch.bfloat16, seed=42)]
    Wa = fv.favor_make_features(5, 256, 64).cuda()
    Wb = fv.favor_make_features(6, 256, 128).cuda()
    first = None
    for it in range(12):
        oa = fv.favor_attention(*a, Wa)
        ob = fv.favor_attention(*b, Wb)
        fv.favor_device_check()
        assert bool(torch.isfinite(oa).all()) and bool(torch.isfinite(ob).all()), it
        if first is None:
            first = (oa.clone(), ob.clone())
        assert torch.equal(oa, first[0]) and torch.equal(ob, first[1]), it


@pytest.mark.parametrize("overlap", [False, True])
@pytest.mark.parametrize("H,Hkv,d", [(8, 8, 64), (8, 1, 128)])
def test_back_to_back_calls_reusing_scratch(H, Hkv, d, overlap):
    # Three stage sequences issued back to back on one stream with no synchronisation, all
    # sharing one partial-state and one state buffer.  With launch overlap on, every kernel may
    # start while the one before it finishes; each must still wait before it overwrites a
    # buffer an earlier kernel reads (the next key pass's partials, the next reduction's state),
    # so every output equals the same call made alone, bit for bit.
    before = fv.favor_set_launch_overlap(overlap)
    try:
        _back_to_back(H, Hkv, d)
    finally:
        fv.favor_set_launch_overlap(before)


def _back_to_back(H, Hkv, d):
    B, L, m = 2, 8192, 256
    W = fv.favor_make_features(3, m, d).cuda()
    sets = [[t.cuda() for t in wl.random_inputs(B, H, Hkv, L, d, torch.bfloat16, seed=20 + i)] for i in range(3)]
    part = torch.empty(fv.favor_partials_bytes(B, Hkv, L, d, m), dtype=torch.uint8, device="cuda")
    state = torch.empty(fv.favor_state_bytes(B, Hkv, d, m), dtype=torch.uint8, device="cuda")
    outs = [torch.empty_like(q) for q, _, _ in sets]
    for (Qd, Kd, Vd), out in zip(sets, outs):
        fv.favor_key_pass(Kd, Vd, W, part)
        fv.favor_state_reduce(part, state, B, Hkv, L, d, m)
        fv.favor_query_pass(Qd, W, state, Hkv, out)
    fv.favor_device_check()
    for (Qd, Kd, Vd), out in zip(sets, outs):
        alone = fv.favor_attention(Qd, Kd, Vd, W)
        fv.favor_device_check()
        assert torch.equal(out, alone)
    assert not torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_stage_calls_equal_fused_call_and_state_matches_oracle(dtype):
    B, H, Hkv, L, d, m = 2, 4, 2, 1500, 64, 192
    Q, K, V = wl.random_inputs(B, H, Hkv, L, d, dtype, seed=11)
    W = fv.favor_make_features(1, m, d)
    Qd, Kd, Vd, Wd = Q.cuda(), K.cuda(), V.cuda(), W.cuda()
    part = torch.empty(fv.favor_partials_bytes(B, Hkv, L, d, m), dtype=torch.uint8, device="cuda")
    state = torch.empty(fv.favor_state_bytes(B, Hkv, d, m), dtype=torch.uint8, device="cuda")
    fv.favor_key_pass(Kd, Vd, Wd, part)
    fv.favor_state_reduce(part, state, B, Hkv, L, d, m)
    out = torch.empty_like(Qd)
    fv.favor_query_pass(Qd, Wd, state, Hkv, out)
    fused = fv.favor_attention(Qd, Kd, Vd, Wd)
    fv.favor_device_check()
    assert torch.equal(out, fused)
    S, _ = fv.state_views(state, B, Hkv, d, m)
    Wo = ofv.make_features_f32(1, m, d)
    # Each key feature carries a relative error of at most eps (bf16: 2^-9 rounding of phi
    # plus ~1e-3 from the exponent argument; fp32: far below 1e-4), so every state entry
    # sum_t phi_t v_t is within eps * sum_t phi_t |v_t| of the exact one.
    eps = 6e-3 if dtype == torch.bfloat16 else 1e-4
    for b in range(B):
        for g in range(Hkv):
            So, _ = ofv.key_state(f64(K[b, g]), f64(V[b, g]), Wo)
            Sa, _ = ofv.key_state(f64(K[b, g]), np.abs(f64(V[b, g])), Wo)
            Sg = S[b * Hkv + g].double().cpu().numpy()
            # the state is defined up to one positive constant (stabiliser, 1/sqrt(m))
            gn, on = Sg / Sg[:, d].sum(), So / So[:, d].sum()
            assert np.all(np.abs(gn - on) <= eps * Sa / So[:, d].sum() + 1e-12), np.abs(gn - on).max()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_host_call_pieces_equal_device_calls(dtype):
    # ten kv heads: the host call splits them into eight pieces of consecutive kv heads (sizes 1
    # and 2, one piece across a batch boundary) and runs each as a problem of its own, so each
    # piece must equal the device call on the same heads bit for bit
    B, H, Hkv, L, d, m = 5, 4, 2, 200, 64, 64
    G, KH, NP = H // Hkv, B * Hkv, 8
    Q, K, V = wl.random_inputs(B, H, Hkv, L, d, dtype, seed=9)
    W = fv.favor_make_features(2, m, d)
    host = fv.favor_attention_host(Q.pin_memory(), K.pin_memory(), V.pin_memory(), W)
    Qf, Kf, Vf, Of = (x.reshape(-1, L, d) for x in (Q, K, V, host))
    spans = []
    for i in range(NP):
        t0, t1 = KH * i // NP, KH * (i + 1) // NP
        spans.append((t0, t1))
        dev = gpu_attention(Qf[t0 * G:t1 * G][None], Kf[t0:t1][None], Vf[t0:t1][None], W)
        assert torch.equal(Of[t0 * G:t1 * G], dev[0].cpu()), (i, t0, t1)
    assert any(t0 // Hkv != (t1 - 1) // Hkv for t0, t1 in spans)  # a piece spans two batches


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_host_call_equals_device_call(dtype):
    Q, K, V = wl.random_inputs(1, 2, 1, 777, 128, dtype, seed=5)
    W = fv.favor_make_features(1, 128, 128)
    host = fv.favor_attention_host(Q.pin_memory(), K.pin_memory(), V.pin_memory(), W)
    dev = gpu_attention(Q, K, V, W)
    assert torch.equal(host, dev)


def test_chained_calls_with_the_default_launch_read_the_previous_output():
    # stacked layers: each call's out is the next call's Q, K and V, issued back to back on one
    # stream.  With the default (ordinary first launch) every call starts after the previous one
    # has completed, so the chain equals the same calls separated by synchronisations.
    before = fv.favor_set_launch_overlap(False)
    try:
        B, H, Hkv, L, d, m = 2, 4, 4, 3000, 64, 256
        x = [t.cuda() for t in wl.random_inputs(B, H, Hkv, L, d, torch.bfloat16, seed=31)][0]
        W = fv.favor_make_features(5, m, d).cuda()
        chain = [x]
        for _ in range(3):
            chain.append(fv.favor_attention(chain[-1], chain[-1], chain[-1], W))
        fv.favor_device_check()
        step = x
        for k in range(3):
            step = fv.favor_attention(step, step, step, W)
            fv.favor_device_check()
            assert torch.equal(chain[k + 1], step), k
    finally:
        fv.favor_set_launch_overlap(before)


@pytest.mark.parametrize("d,m", [(64, 256), (64, 128), (128, 256)])
def test_many_short_heads(d, m):
    # many heads of one or two query tiles each: every CTA walks several kv heads, and each of its
    # two epilogue warpgroups skips the kv heads whose tiles all went to the other one
    for L in (100, 200):
        Q, K, V = wl.random_inputs(8, 96, 96, L, d, torch.bfloat16, seed=L + d)
        run_case(Q, K, V, m, what=f"L={L} d={d} m={m}")
