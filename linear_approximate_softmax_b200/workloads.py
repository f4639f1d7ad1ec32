"""Seeded synthetic inputs for FAVOR+ attention.

This module only draws random numbers; it holds none of the method's
arithmetic, so both the CUDA path's tests and the oracle can consume what it
returns.  The five workloads stand in for the long-sequence tasks that
"Rethinking Attention with Performers" (Abstract; 주요 결과 / main results)
and "Fast Transformer Decoding: One Write-Head is All You Need" (multi-query
layout) evaluate on; those datasets are not used.

Draw order under ``torch.Generator('cpu').manual_seed(data_seed)``:
Q [B,H,L,d], K [B,Hkv,L,d], V [B,Hkv,L,d] (standard normal, fp32), then, for
workloads with heavy-tailed keys, one lognormal(0, sigma) factor per key row
([B,Hkv,L,1]).  Scale factors apply before the cast to the workload dtype.
"""
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: torch.dtype
    B: int
    H: int
    Hkv: int
    L: int
    d: int
    m: int
    qk_scale: float = 1.0
    key_lognormal_sigma: float = 0.0
    orthogonal: tuple = (True,)
    data_seed: int = 0
    w_seed: int = 1

    @property
    def units(self):
        """Token-query-head pairs per pass: B * H * L."""
        return self.B * self.H * self.L


WORKLOADS = {
    "fp32_L256": Workload("fp32_L256", torch.float32, 1, 1, 1, 256, 64, 128),
    "bf16_L4096": Workload("bf16_L4096", torch.bfloat16, 8, 8, 8, 4096, 64, 256, qk_scale=0.5),
    "bf16_L16384_heavykeys": Workload("bf16_L16384_heavykeys", torch.bfloat16, 4, 12, 12, 16384, 64, 256,
                                      key_lognormal_sigma=0.5),
    "bf16_mqa_L8192_d128": Workload("bf16_mqa_L8192_d128", torch.bfloat16, 16, 16, 1, 8192, 128, 256),
    "bf16_L131072_m512": Workload("bf16_L131072_m512", torch.bfloat16, 1, 8, 8, 131072, 64, 512,
                                  orthogonal=(True, False)),
}
WORKLOAD_ORDER = list(WORKLOADS)


def make_inputs(w: Workload, B=None, H=None, Hkv=None, L=None):
    """Q, K, V on the CPU in the workload dtype (optionally at reduced sizes)."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    Hkv = w.Hkv if Hkv is None else Hkv
    L = w.L if L is None else L
    g = torch.Generator("cpu").manual_seed(w.data_seed)
    Q = torch.randn(B, H, L, w.d, generator=g)
    K = torch.randn(B, Hkv, L, w.d, generator=g)
    V = torch.randn(B, Hkv, L, w.d, generator=g)
    if w.qk_scale != 1.0:
        Q.mul_(w.qk_scale)
        K.mul_(w.qk_scale)
    if w.key_lognormal_sigma:
        K.mul_(torch.exp(w.key_lognormal_sigma * torch.randn(B, Hkv, L, 1, generator=g)))
    return Q.to(w.dtype), K.to(w.dtype), V.to(w.dtype)


def random_inputs(B, H, Hkv, L, d, dtype, seed=0, scale=1.0):
    """Plain N(0, scale^2) Q, K and N(0, 1) V for shape-sweep tests."""
    g = torch.Generator("cpu").manual_seed(seed)
    Q = torch.randn(B, H, L, d, generator=g) * scale
    K = torch.randn(B, Hkv, L, d, generator=g) * scale
    V = torch.randn(B, Hkv, L, d, generator=g)
    return Q.to(dtype), K.to(dtype), V.to(dtype)
