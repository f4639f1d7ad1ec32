"""The C-ABI library loads, exports what include/*.h declares, and rejects bad
arguments on the host without launching anything (no GPU needed)."""
import ctypes
import glob
import os
import re

import numpy as np
import pytest
import torch

import linear_approximate_softmax_b200 as fv
from oracle import favor as ofv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names.update(re.findall(r"FAVOR_API\s+[\w\s\*]+?\b(favor_\w+)\s*\(", src))
    return sorted(names)


def test_header_declares_the_api():
    names = declared_symbols()
    assert "favor_attention" in names and "favor_make_features" in names
    assert set(fv.EXPORTS) <= set(names)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(fv.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_version():
    assert fv.favor_version() >= 100


@pytest.mark.parametrize("seed,m,d,orth", [(1, 128, 64, True), (1, 256, 64, True), (1, 256, 128, True),
                                           (1, 512, 64, True), (1, 512, 64, False), (9, 100, 16, True),
                                           (2**63 + 5, 48, 128, False)])
def test_make_features_matches_oracle(seed, m, d, orth):
    got = fv.favor_make_features(seed, m, d, orth).numpy()
    want = ofv.make_features_f32(seed, m, d, orth)
    # both round the same fp64 construction to fp32; allow one fp32 ulp for libm differences
    np.testing.assert_array_max_ulp(got, want, maxulp=1)


def test_make_features_rejects_bad_arguments():
    assert fv.lib.favor_make_features(1, 16, 16, 1, None) == fv.FAVOR_ERR_INVALID
    buf = torch.empty(16)
    assert fv.lib.favor_make_features(1, 0, 16, 1, ctypes.c_void_p(buf.data_ptr())) == fv.FAVOR_ERR_INVALID
    assert fv.lib.favor_make_features(1, 4, 0, 1, ctypes.c_void_p(buf.data_ptr())) == fv.FAVOR_ERR_INVALID
    assert b"favor_make_features" in fv.lib.favor_last_error()


FAKE = 0x1000_0000  # 16-byte aligned; never dereferenced: every case below fails before any launch


def attn(ptrs, B=1, H=1, Hkv=1, L=16, d=64, m=64):
    return fv.lib.favor_attention(*[ctypes.c_void_p(p) for p in ptrs], B, H, Hkv, L, d, m, None)


@pytest.mark.parametrize("shape,code", [
    (dict(d=32), fv.FAVOR_ERR_UNSUPPORTED),
    (dict(d=96), fv.FAVOR_ERR_UNSUPPORTED),
    (dict(m=8), fv.FAVOR_ERR_UNSUPPORTED),
    (dict(m=520), fv.FAVOR_ERR_UNSUPPORTED),
    (dict(m=72), fv.FAVOR_ERR_UNSUPPORTED),
    (dict(H=3, Hkv=2), fv.FAVOR_ERR_UNSUPPORTED),
    (dict(L=0), fv.FAVOR_ERR_UNSUPPORTED),
    (dict(B=0), fv.FAVOR_ERR_UNSUPPORTED),
    (dict(B=4096, H=16, Hkv=16), fv.FAVOR_ERR_UNSUPPORTED),  # B * H above the grid limit
])
def test_attention_rejects_unsupported_shapes(shape, code):
    assert attn([FAKE] * 5, **shape) == code
    assert fv.lib.favor_last_error()


def test_launch_overlap_setting_round_trips():
    before = fv.favor_set_launch_overlap(True)
    try:
        assert fv.favor_set_launch_overlap(False) is True
        assert fv.favor_set_launch_overlap(False) is False
        assert fv.lib.favor_set_launch_overlap(7) == 0 and fv.lib.favor_set_launch_overlap(0) == 1
    finally:
        fv.favor_set_launch_overlap(before)


def test_attention_rejects_null_and_misaligned_pointers():
    assert attn([FAKE, 0, FAKE, FAKE, FAKE]) == fv.FAVOR_ERR_INVALID
    assert attn([FAKE, FAKE, FAKE + 8, FAKE, FAKE]) == fv.FAVOR_ERR_INVALID
    assert b"aligned" in fv.lib.favor_last_error()


def test_stage_calls_reject_bad_dtype_and_pointers():
    p = ctypes.c_void_p(FAKE)
    assert fv.lib.favor_key_pass(7, p, p, p, p, 1, 1, 16, 64, 64, None) == fv.FAVOR_ERR_INVALID
    assert fv.lib.favor_query_pass(fv.FAVOR_BF16, p, None, p, p, 1, 1, 1, 16, 64, 64, None) == fv.FAVOR_ERR_INVALID
    assert fv.lib.favor_state_reduce(p, None, 1, 1, 16, 64, 64, None) == fv.FAVOR_ERR_INVALID
    assert fv.lib.favor_attention_host(5, p, p, p, p, p, 1, 1, 1, 16, 64, 64, None) == fv.FAVOR_ERR_INVALID


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_valid_call_without_a_device_reports_cuda_error():
    assert attn([FAKE] * 5) == fv.FAVOR_ERR_CUDA
    assert fv.favor_partials_bytes(1, 1, 16, 64, 64) == 0
    # the host-buffer call fails cleanly before it copies anything
    q = np.zeros(16 * 64, np.uint16)
    w = np.zeros(64 * 64, np.float32)
    ptr = lambda x: ctypes.c_void_p(x.ctypes.data)  # noqa: E731
    rc = fv.lib.favor_attention_host(fv.FAVOR_BF16, ptr(q), ptr(q), ptr(q), ptr(w), ptr(q.copy()), 1, 1, 1, 16, 64, 64, None)
    assert rc == fv.FAVOR_ERR_CUDA and fv.lib.favor_last_error()


def test_decode_state_bytes_and_argument_errors():
    # per kv head: S [m][d+1] and c [m], fp32
    assert fv.favor_decode_state_bytes(2, 1, 128, 256) == 2 * 1 * 256 * 130 * 4
    assert fv.favor_decode_state_bytes(1, 3, 64, 16) == 3 * 16 * 66 * 4
    assert fv.favor_decode_state_bytes(1, 1, 96, 256) == 0   # unsupported d
    assert fv.favor_decode_state_bytes(1, 1, 64, 520) == 0   # m above 512
    p = ctypes.c_void_p(FAKE)
    lib = fv.lib
    assert lib.favor_decode_step(7, p, p, p, p, p, p, 1, 2, 2, 64, 128, None) == fv.FAVOR_ERR_INVALID
    assert lib.favor_decode_step(0, p, p, p, p, p, p, 1, 3, 2, 64, 128, None) == fv.FAVOR_ERR_UNSUPPORTED
    assert lib.favor_decode_step(0, p, p, p, p, p, p, 1, 65, 1, 64, 128, None) == fv.FAVOR_ERR_UNSUPPORTED
    assert lib.favor_decode_step(0, None, p, p, p, p, p, 1, 2, 2, 64, 128, None) == fv.FAVOR_ERR_INVALID
    assert lib.favor_decode_init(ctypes.c_void_p(FAKE + 8), 1, 1, 64, 128, None) == fv.FAVOR_ERR_INVALID
