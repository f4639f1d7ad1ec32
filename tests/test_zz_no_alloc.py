"""favor_attention_noalloc: same results as favor_attention, with no allocation.

Callers whose device memory is owned by their own allocator, or whose serving
loop cannot afford an allocator call, use favor_attention_noalloc; it keeps
its scratch in a static array inside the library.  This file is named so that
pytest collects it last; it must pass on its own in a fresh process and after
every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import linear_approximate_softmax_b200 as fv  # noqa: E402
from linear_approximate_softmax_b200 import workloads as wl  # noqa: E402

TOL = {torch.bfloat16: (2e-2, 5e-3), torch.float32: (1e-4, 1e-4)}


def _noalloc(Q, K, V, W):
    """One call through the C ABI, on the current stream."""
    B, H, L, d = Q.shape
    out = torch.empty_like(Q)
    code = fv.FAVOR_BF16 if Q.dtype == torch.bfloat16 else fv.FAVOR_F32
    rc = fv.lib.favor_attention_noalloc(
        code, ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(K.data_ptr()), ctypes.c_void_p(V.data_ptr()),
        ctypes.c_void_p(W.data_ptr()), ctypes.c_void_p(out.data_ptr()), B, H, K.shape[1], L, d, W.shape[0],
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == fv.FAVOR_OK, fv.lib.favor_last_error()
    return out


def _close(got, ref, dtype):
    g = got.float().cpu().numpy().astype(np.float64)
    r = ref.float().cpu().numpy().astype(np.float64)
    diff = np.abs(g - r)
    tol_abs, tol_rel = TOL[dtype]
    assert np.all(np.isfinite(g))
    assert diff.max() <= tol_abs and diff.sum() / np.abs(r).sum() <= tol_rel, (diff.max(), diff.sum() / np.abs(r).sum())


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_two_calls_in_a_row_match_the_allocating_call(dtype):
    # the headline shape keeps more key chunks than fit, so the scratch layout is re-split
    shapes = [(4, 12, 12, 16384, 64, 256), (2, 8, 1, 3001, 128, 192)]
    for i, (B, H, Hkv, L, d, m) in enumerate(shapes):
        Q, K, V = [t.cuda() for t in wl.random_inputs(B, H, Hkv, L, d, dtype, seed=40 + i)]
        W = fv.favor_make_features(1 + i, m, d).cuda()
        ref = fv.favor_attention(Q, K, V, W)
        got = _noalloc(Q, K, V, W)
        torch.cuda.synchronize()
        _close(got, ref, dtype)


def test_second_call_does_not_see_the_first_calls_scratch():
    Q1, K1, V1 = [t.cuda() for t in wl.random_inputs(1, 2, 1, 2000, 64, torch.bfloat16, seed=1)]
    Q2, K2, V2 = [t.cuda() for t in wl.random_inputs(1, 2, 1, 700, 64, torch.bfloat16, seed=2)]
    W = fv.favor_make_features(3, 128, 64).cuda()
    a = _noalloc(Q1, K1, V1, W)
    b = _noalloc(Q2, K2, V2, W)
    torch.cuda.synchronize()
    _close(a, fv.favor_attention(Q1, K1, V1, W), torch.bfloat16)
    _close(b, fv.favor_attention(Q2, K2, V2, W), torch.bfloat16)


def test_shape_beyond_the_static_scratch_is_rejected():
    # 64 kv heads x m=512 x (d+1)=129 fp32 state alone is 17 MB, more than the 16 MiB array
    p = ctypes.c_void_p(0x1000_0000)
    rc = fv.lib.favor_attention_noalloc(fv.FAVOR_BF16, p, p, p, p, p, 1, 64, 64, 128, 128, 512, None)
    assert rc == fv.FAVOR_ERR_UNSUPPORTED
    assert b"static scratch" in fv.lib.favor_last_error()
