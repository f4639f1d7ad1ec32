"""FAVOR+ attention on B200 (sm_100a): Python binding of libfavor_b200.so.

Every function here only marshals arguments (tensor pointers, sizes, the
current CUDA stream) into the C ABI declared in include/favor.h; all of the
arithmetic runs in the library's CUDA kernels.  PyTorch supplies device memory
and streams.  The names match the C entry points.

The library must have been built (``python linear_approximate_softmax_b200/build.py``);
importing this package without it raises ImportError — there is no fallback.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfavor_b200.so")

FAVOR_OK = 0
FAVOR_ERR_INVALID = -1
FAVOR_ERR_UNSUPPORTED = -2
FAVOR_ERR_CUDA = -3
FAVOR_ERR_NOMEM = -4
FAVOR_ERR_TIMEOUT = -5
FAVOR_BF16 = 0
FAVOR_F32 = 1

EXPORTS = [
    "favor_last_error", "favor_version", "favor_make_features", "favor_attention",
    "favor_attention_f32", "favor_attention_host", "favor_partials_bytes", "favor_state_bytes",
    "favor_key_pass", "favor_state_reduce", "favor_query_pass", "favor_attention_noalloc", "favor_device_check",
    "favor_set_launch_overlap", "favor_decode_state_bytes", "favor_decode_init", "favor_decode_step",
    "favor_attention_relu", "favor_linformer",
]

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python linear_approximate_softmax_b200/build.py`")
lib = ctypes.CDLL(LIB_PATH)

_i, _p, _sz, _u64 = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint64
lib.favor_last_error.restype = ctypes.c_char_p
lib.favor_last_error.argtypes = []
lib.favor_version.restype = _i
lib.favor_make_features.argtypes = [_u64, _i, _i, _i, _p]
lib.favor_make_features.restype = _i
_ATT = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _p]
lib.favor_attention.argtypes = _ATT
lib.favor_attention.restype = _i
lib.favor_attention_f32.argtypes = _ATT
lib.favor_attention_f32.restype = _i
lib.favor_attention_host.argtypes = [_i] + _ATT
lib.favor_attention_host.restype = _i
lib.favor_attention_relu.argtypes = [_i] + _ATT
lib.favor_attention_relu.restype = _i
lib.favor_linformer.argtypes = [_i, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _p]
lib.favor_linformer.restype = _i
lib.favor_partials_bytes.argtypes = [_i, _i, _i, _i, _i]
lib.favor_partials_bytes.restype = _sz
lib.favor_state_bytes.argtypes = [_i, _i, _i, _i]
lib.favor_state_bytes.restype = _sz
lib.favor_key_pass.argtypes = [_i, _p, _p, _p, _p, _i, _i, _i, _i, _i, _p]
lib.favor_key_pass.restype = _i
lib.favor_state_reduce.argtypes = [_p, _p, _i, _i, _i, _i, _i, _p]
lib.favor_state_reduce.restype = _i
lib.favor_query_pass.argtypes = [_i, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _p]
lib.favor_query_pass.restype = _i
lib.favor_device_check.argtypes = [_p]
lib.favor_device_check.restype = _i
lib.favor_attention_noalloc.argtypes = [_i] + _ATT
lib.favor_attention_noalloc.restype = _i
lib.favor_set_launch_overlap.argtypes = [_i]
lib.favor_set_launch_overlap.restype = _i
lib.favor_decode_state_bytes.argtypes = [_i, _i, _i, _i]
lib.favor_decode_state_bytes.restype = _sz
lib.favor_decode_init.argtypes = [_p, _i, _i, _i, _i, _p]
lib.favor_decode_init.restype = _i
lib.favor_decode_step.argtypes = [_i, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _p]
lib.favor_decode_step.restype = _i


def favor_set_launch_overlap(enable):
    """Whether the first kernel of each later call may start while the kernel before it on the
    stream finishes (see favor.h); returns the previous setting."""
    return bool(lib.favor_set_launch_overlap(1 if enable else 0))


class FavorError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__(f"{where} failed ({code}): {lib.favor_last_error().decode(errors='replace')}")


def _check(rc, where):
    if rc != FAVOR_OK:
        raise FavorError(rc, where)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return FAVOR_BF16
    if t.dtype == torch.float32:
        return FAVOR_F32
    raise TypeError(f"unsupported dtype {t.dtype}; use torch.bfloat16 or torch.float32")


def _dev(t, name):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    return ctypes.c_void_p(t.data_ptr())


def _shape(Q, K, V, W):
    B, H, L, d = Q.shape
    if K.dim() != 4 or K.shape[0] != B or K.shape[2] != L or K.shape[3] != d or V.shape != K.shape:
        raise ValueError(f"K, V must be [B, Hkv, L, d] matching Q {tuple(Q.shape)}; got {tuple(K.shape)}, {tuple(V.shape)}")
    if W.dim() != 2 or W.shape[1] != d:
        raise ValueError(f"W must be [m, {d}], got {tuple(W.shape)}")
    return B, H, K.shape[1], L, d, W.shape[0]


def favor_version():
    return lib.favor_version()


def favor_device_check(stream=None):
    """Synchronise the stream and raise FavorError if a GPU kernel gave up waiting."""
    _check(lib.favor_device_check(_stream(stream)), "favor_device_check")


def favor_make_features(seed, m, d, orthogonal=True):
    """W [m, d] fp32 on the host (see favor_make_features in include/favor.h)."""
    W = torch.empty(m, d, dtype=torch.float32)
    _check(lib.favor_make_features(int(seed), int(m), int(d), int(bool(orthogonal)), ctypes.c_void_p(W.data_ptr())),
           "favor_make_features")
    return W


def favor_attention(Q, K, V, W, out=None, stream=None):
    """FAVOR+ attention on device tensors; bf16 or fp32 (Q, K, V, out share the dtype)."""
    code = _dtype_code(Q)
    if K.dtype != Q.dtype or V.dtype != Q.dtype or W.dtype != torch.float32:
        raise TypeError("Q, K, V must share a dtype and W must be float32")
    B, H, Hkv, L, d, m = _shape(Q, K, V, W)
    if out is None:
        out = torch.empty_like(Q)
    fn = lib.favor_attention if code == FAVOR_BF16 else lib.favor_attention_f32
    _check(fn(_dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), _dev(W, "W"), _dev(out, "out"), B, H, Hkv, L, d, m,
              _stream(stream)), fn.__name__)
    return out


favor_attention_f32 = favor_attention


def favor_attention_relu(Q, K, V, W, out=None, stream=None):
    """Kernelizable attention with phi = ReLU(W x') on device tensors; bf16 or fp32."""
    code = _dtype_code(Q)
    if K.dtype != Q.dtype or V.dtype != Q.dtype or W.dtype != torch.float32:
        raise TypeError("Q, K, V must share a dtype and W must be float32")
    B, H, Hkv, L, d, m = _shape(Q, K, V, W)
    if out is None:
        out = torch.empty_like(Q)
    _check(lib.favor_attention_relu(code, _dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), _dev(W, "W"), _dev(out, "out"),
                                    B, H, Hkv, L, d, m, _stream(stream)), "favor_attention_relu")
    return out


def favor_linformer(Q, K, V, E, F, out=None, stream=None):
    """Linformer projected attention on device tensors: E, F are float32 [kp, L] projections."""
    code = _dtype_code(Q)
    if K.dtype != Q.dtype or V.dtype != Q.dtype or E.dtype != torch.float32 or F.dtype != torch.float32:
        raise TypeError("Q, K, V must share a dtype and E, F must be float32")
    if Q.dim() != 4 or K.dim() != 4 or V.shape != K.shape or E.dim() != 2 or E.shape != F.shape:
        raise ValueError("expected Q [B,H,L,d], K and V [B,Hkv,L,d], E and F [kp,L]")
    B, H, L, d = Q.shape
    Hkv, kp = K.shape[1], E.shape[0]
    if K.shape[0] != B or K.shape[2] != L or K.shape[3] != d or E.shape[1] != L:
        raise ValueError("Q, K, V, E, F disagree on B, L or d")
    if out is None:
        out = torch.empty_like(Q)
    _check(lib.favor_linformer(code, _dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), _dev(E, "E"), _dev(F, "F"),
                               _dev(out, "out"), B, H, Hkv, L, d, kp, _stream(stream)), "favor_linformer")
    return out


def favor_attention_host(Q, K, V, W, out=None, stream=None):
    """End-to-end call on host tensors: copies in, computes on the GPU, copies out, syncs."""
    code = _dtype_code(Q)
    for t, n in ((Q, "Q"), (K, "K"), (V, "V"), (W, "W")):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous host tensor")
    B, H, Hkv, L, d, m = _shape(Q, K, V, W)
    if out is None:
        out = torch.empty_like(Q)
    _check(lib.favor_attention_host(code, ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(K.data_ptr()),
                                    ctypes.c_void_p(V.data_ptr()), ctypes.c_void_p(W.data_ptr()),
                                    ctypes.c_void_p(out.data_ptr()), B, H, Hkv, L, d, m, _stream(stream)),
           "favor_attention_host")
    return out


def favor_attention_noalloc(Q, K, V, W, out=None, stream=None):
    """favor_attention without any device allocation (scratch in the library's static array)."""
    code = _dtype_code(Q)
    B, H, Hkv, L, d, m = _shape(Q, K, V, W)
    if out is None:
        out = torch.empty_like(Q)
    _check(lib.favor_attention_noalloc(code, _dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), _dev(W, "W"),
                                       _dev(out, "out"), B, H, Hkv, L, d, m, _stream(stream)),
           "favor_attention_noalloc")
    return out


def favor_partials_bytes(B, Hkv, L, d, m):
    return int(lib.favor_partials_bytes(B, Hkv, L, d, m))


def favor_state_bytes(B, Hkv, d, m):
    return int(lib.favor_state_bytes(B, Hkv, d, m))


def favor_key_pass(K, V, W, partials, stream=None):
    B, Hkv, L, d = K.shape
    _check(lib.favor_key_pass(_dtype_code(K), _dev(K, "K"), _dev(V, "V"), _dev(W, "W"), _dev(partials, "partials"),
                              B, Hkv, L, d, W.shape[0], _stream(stream)), "favor_key_pass")


def favor_state_reduce(partials, state, B, Hkv, L, d, m, stream=None):
    _check(lib.favor_state_reduce(_dev(partials, "partials"), _dev(state, "state"), B, Hkv, L, d, m,
                                  _stream(stream)), "favor_state_reduce")


def favor_query_pass(Q, W, state, Hkv, out, stream=None):
    B, H, L, d = Q.shape
    _check(lib.favor_query_pass(_dtype_code(Q), _dev(Q, "Q"), _dev(W, "W"), _dev(state, "state"), _dev(out, "out"),
                                B, H, Hkv, L, d, W.shape[0], _stream(stream)), "favor_query_pass")
    return out


def favor_decode_state_bytes(B, Hkv, d, m):
    return int(lib.favor_decode_state_bytes(B, Hkv, d, m))


def favor_decode_init(state, B, Hkv, d, m, stream=None):
    """Empty decode state (uint8 CUDA tensor of favor_decode_state_bytes(...) bytes)."""
    _check(lib.favor_decode_init(_dev(state, "state"), B, Hkv, d, m, _stream(stream)), "favor_decode_init")
    return state


def favor_decode_step(q, k, v, W, state, out=None, stream=None):
    """One decoding step: q [B, H, d], k, v [B, Hkv, d] device tensors; updates `state` in place."""
    code = _dtype_code(q)
    B, H, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, d) or v.shape != k.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError(f"k, v must be [B, Hkv, d] of q's dtype; got {tuple(k.shape)}, {tuple(v.shape)}")
    if out is None:
        out = torch.empty_like(q)
    _check(lib.favor_decode_step(code, _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(W, "W"), _dev(state, "state"),
                                 _dev(out, "out"), B, H, Hkv, d, W.shape[0], _stream(stream)), "favor_decode_step")
    return out


def state_views(state, B, Hkv, d, m):
    """Views of the public part of a state buffer (uint8 CUDA tensor): S [B*Hkv, m, d+1] and c [B*Hkv]."""
    D1 = d + 1
    heads = B * Hkv
    s_bytes = heads * m * D1 * 4
    c_off = (s_bytes + 255) // 256 * 256
    S = state[:s_bytes].view(torch.float32).view(heads, m, D1)
    c = state[c_off:c_off + heads * 4].view(torch.float32)
    return S, c
