// FAVOR+ on CUDA cores: fp32 arithmetic throughout, fp32 or bf16 storage.
//
// This is the exact-arithmetic path (the fp32 entry point) and the reference
// GPU path for bf16 inputs.  Three kernels, one per step of the linear-time
// estimate ("Rethinking Attention with Performers", Abstract: linear space and
// time; 제안 방법: positive random features):
//
//   key pass     per (kv head, key chunk, 64-feature block):
//                u = W'k - n(k) (log2 units), chunk max stabiliser c (running,
//                with exact rescaling of the accumulator when it grows),
//                S_part = sum_t 2^(u_t - c) [v_t | 1]
//   reduce       per kv head: c* = max c, S = sum_p 2^(c_p - c*) S_p in chunk order
//   query pass   per (query head, 32-query tile): u = W'q, per-row max
//                stabiliser, out = (phi S[:, :d]) / (phi S[:, d])
//
// W' = d^-1/4 log2(e) W and n(k) = d^-1/2 log2(e) |k|^2 / 2, so 2^(W'k - n(k))
// = exp(W k' - |k'|^2/2) with k' = d^-1/4 k.  The query's -|q'|^2/2 term and
// the 1/sqrt(m) factors are constant along a query row and cancel exactly in
// the ratio, as any per-row stabiliser does; they are not computed.
//
// The key and query kernels also serve the generalised kernelizable attention
// of the same page (Abstract; 연구 질문 RQ5) with f = ReLU: phi = max(W'x, 0) with
// W' = d^-1/4 W, no norm term and no stabiliser (phi >= 0 is bounded by |W'x|; the
// chunk stabilisers are written as 0, so the reduction sums the chunks as they are).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "favor_internal.h"
#include "launch.cuh"

namespace favor {
namespace {

constexpr int kThreads = 256;
constexpr int kFB = 64;   // features per key-pass CTA
constexpr int kTT = 32;   // tokens per key-pass step
constexpr int kQT = 32;   // queries per query-pass CTA
constexpr int kExp = 0;   // feature maps: FAVOR+ positive features (exp)
constexpr int kRelu = 1;  //               max(W'x, 0)

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void store_as(float* p, float x) { *p = x; }
__device__ __forceinline__ void store_as(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// grid (P, B*Hkv, ceil(m/64)), 256 threads.  One running stabiliser per CTA,
// written for each of its features (0 for f = ReLU).
template <typename T, int D, int FMAP>
__global__ void __launch_bounds__(kThreads) key_pass_kernel(
    const T* __restrict__ K, const T* __restrict__ V, const float* __restrict__ W,
    float* __restrict__ part_S, float* __restrict__ part_c, int L, int m, int P, int chunk,
    int nsb, float wscale, float nscale) {
  constexpr int D1 = D + 1;
  constexpr int NE = (kFB * D1 + kThreads - 1) / kThreads;
  extern __shared__ float smem[];
  float* Ws = smem;                  // [kFB][D1]   (row stride D1 keeps banks apart)
  float* Ks = Ws + kFB * D1;         // [kTT][D1]   column D holds n(k)
  float* Vs = Ks + kTT * D1;         // [kTT][D1]   column D holds 1 (0 past the end)
  float* U = Vs + kTT * D1;          // [kTT][kFB+1]
  float* red = U + kTT * (kFB + 1);  // [kThreads/32]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int p = blockIdx.x, head = blockIdx.y, fb = blockIdx.z;
  const int f0 = fb * kFB, fbw = min(kFB, m - f0);
  const int t_begin = p * chunk, t_end = min(L, t_begin + chunk);
  const T* Kh = K + static_cast<size_t>(head) * L * D;
  const T* Vh = V + static_cast<size_t>(head) * L * D;

  for (int i = tid; i < kFB * D; i += kThreads) {
    const int f = i / D, j = i % D;
    Ws[f * D1 + j] = f < fbw ? W[static_cast<size_t>(f0 + f) * D + j] * wscale : 0.f;
  }

  float acc[NE];
#pragma unroll
  for (int k = 0; k < NE; ++k) acc[k] = 0.f;
  float c_run = -INFINITY;

  for (int t0 = t_begin; t0 < t_end; t0 += kTT) {
    const int tw = min(kTT, t_end - t0);
    __syncthreads();  // previous step is done with Ks, Vs, U, red
    for (int i = tid; i < kTT * D; i += kThreads) {
      const int t = i / D, j = i % D;
      float kv = 0.f, vv = 0.f;
      if (t < tw) {
        kv = to_f32(Kh[static_cast<size_t>(t0 + t) * D + j]);
        vv = to_f32(Vh[static_cast<size_t>(t0 + t) * D + j]);
      }
      Ks[t * D1 + j] = kv;
      Vs[t * D1 + j] = vv;
    }
    if (tid < kTT) Vs[tid * D1 + D] = tid < tw ? 1.f : 0.f;
    __syncthreads();
    if (tid < kTT) {
      float s = 0.f;
      if (FMAP == kExp)
        for (int j = 0; j < D; ++j) s = fmaf(Ks[tid * D1 + j], Ks[tid * D1 + j], s);
      Ks[tid * D1 + D] = s * nscale;
    }
    __syncthreads();

    float lmax = -INFINITY;
    for (int i = tid; i < kTT * kFB; i += kThreads) {
      const int t = i / kFB, f = i % kFB;
      float u = -INFINITY;
      if (t < tw && f < fbw) {
        float s = 0.f;
#pragma unroll 16
        for (int j = 0; j < D; ++j) s = fmaf(Ks[t * D1 + j], Ws[f * D1 + j], s);
        u = s - Ks[t * D1 + D];
      }
      U[t * (kFB + 1) + f] = u;
      lmax = fmaxf(lmax, u);
    }
    float rescale = 1.f;
    if (FMAP == kExp) {
      lmax = warp_max(lmax);
      if (lane == 0) red[warp] = lmax;
      __syncthreads();
      float tmax = red[0];
#pragma unroll
      for (int w = 1; w < kThreads / 32; ++w) tmax = fmaxf(tmax, red[w]);
      const float c_new = fmaxf(c_run, tmax);
      rescale = (c_run == -INFINITY) ? 1.f : exp2f(c_run - c_new);
      c_run = c_new;
    } else {
      c_run = 0.f;
    }
    for (int i = tid; i < kTT * kFB; i += kThreads) {
      const int t = i / kFB, f = i % kFB;
      const float u = U[t * (kFB + 1) + f];
      U[t * (kFB + 1) + f] = FMAP == kExp ? ((u == -INFINITY) ? 0.f : exp2f(u - c_run)) : fmaxf(u, 0.f);
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < NE; ++k) {
      const int e = tid + k * kThreads;
      if (e < kFB * D1) {
        const int f = e / D1, c = e % D1;
        float a = acc[k] * rescale;
        for (int t = 0; t < tw; ++t) a = fmaf(U[t * (kFB + 1) + f], Vs[t * D1 + c], a);
        acc[k] = a;
      }
    }
  }

  float* out = part_S + (static_cast<size_t>(head) * P + p) * static_cast<size_t>(m) * D1;
#pragma unroll
  for (int k = 0; k < NE; ++k) {
    const int e = tid + k * kThreads;
    if (e < kFB * D1) {
      const int f = e / D1, c = e % D1;
      if (f < fbw) out[static_cast<size_t>(f0 + f) * D1 + c] = acc[k];
    }
  }
  if (FMAP == kRelu) c_run = 0.f;  // no token in this chunk: still no stabiliser
  for (int f = tid; f < fbw; f += kThreads) part_c[(static_cast<size_t>(head) * P + p) * nsb + f0 + f] = c_run;
}

// grid (op_tail / 32, B*Hkv), 256 threads: 32 feature rows per CTA, 8 threads
// per row.  Each row is the sum of the chunk partials in the fixed order p = 0..P-1,
// each rescaled from its own stabiliser to the row's largest one c_f (bitwise
// deterministic).  Writes S[f][n] = 2^(c_f - c*) x that sum (fp32, relative to the head's
// largest stabiliser c*), c*, and the fp16 operand image of the query pass: the row
// relative to c_f scaled by 2^-x_f so that its largest entry lies in [2^14, 2^15), then
// e_f = x_f + (c_f - c*) and the normaliser entry with the same scaling.  Because the
// image carries c_f - c* in e_f rather than in its fp16 values, a feature whose keys sit
// far below the head's largest exponent keeps its precision on the query side.
// The kernel is latency-bound: the rows of CB chunks, the feature's stabilisers and the
// head's stabilisers are all requested before any of them is used, and the image goes out
// through shared memory as whole 16-byte pieces of its rows.
template <int D>
__global__ void __launch_bounds__(kThreads, D == 64 ? 4 : 2) state_reduce_kernel(
    const float* __restrict__ part_S, const float* __restrict__ part_c, float* __restrict__ S,
    float* __restrict__ Sc, unsigned char* __restrict__ op, int P, int m, int nsb, int op_atoms, int op_tail,
    size_t op_bytes, int op_rows) {
  constexpr int D1 = D + 1;
  constexpr int NC = (D1 + 7) / 8;     // columns per thread: g, g + 8, ...
  constexpr int CB = D == 64 ? 3 : 2;  // chunks whose rows are in flight together
  __shared__ float red[kThreads / 32];
  // the image rows of this CTA's 32 features: D outputs, then (when the image has D + 16 rows)
  // the normaliser row and 15 rows of zeros
  __shared__ __align__(16) __half stage[D + 16][32];
  griddep_launch_dependents();
  griddep_wait();  // the partial state comes from the kernel before this one on the stream
  // That kernel may still have been writing the partial state while this one was already
  // resident (programmatic launch), so it is read with loads cached in L2 only (__ldcg), never
  // through the read-only path, which may serve lines from before the writes.
  const int head = blockIdx.y, tid = threadIdx.x;
  const int fl = tid >> 3, f0 = blockIdx.x * 32, f = f0 + fl;  // feature row (< op_tail)
  const int g = tid & 7;
  const bool live = f < m;
  const float* pc = part_c + static_cast<size_t>(head) * P * nsb;
  const float* rows = part_S + (static_cast<size_t>(head) * P * m + f) * D1;  // chunk p at + p * m * D1
  float x[CB][NC], cc[CB];
  auto load = [&](int p0) {  // CB chunks' rows of this feature and their stabilisers, all in flight at once
#pragma unroll
    for (int b = 0; b < CB; ++b) {
      cc[b] = live && p0 + b < P ? __ldcg(pc + (p0 + b) * nsb + f / kStabBlock) : -INFINITY;
#pragma unroll
      for (int k = 0; k < NC; ++k) {
        const int n = g + 8 * k;
        x[b][k] = live && p0 + b < P && n < D1 ? __ldcg(rows + static_cast<size_t>(p0 + b) * m * D1 + n) : 0.f;
      }
    }
  };
  load(0);
  // the stabiliser maxima, eight independent loads in flight at a time
  float cf = -INFINITY;  // this feature's largest chunk stabiliser
  if (live)
    for (int p0 = 0; p0 < P; p0 += 8) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = p0 + u < P ? __ldcg(pc + (p0 + u) * nsb + f / kStabBlock) : -INFINITY;
#pragma unroll
      for (int u = 0; u < 8; ++u) cf = fmaxf(cf, v[u]);
    }
  float cs = -INFINITY;  // the head's largest stabiliser: 16-byte loads, eight in flight (nsb % 4 == 0)
  {
    const float4* pc4 = reinterpret_cast<const float4*>(pc);
    const int n4 = P * nsb / 4;
    for (int i0 = tid; i0 < n4; i0 += 8 * kThreads) {
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        v[u] = i0 + u * kThreads < n4 ? __ldcg(pc4 + i0 + u * kThreads) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
#pragma unroll
      for (int u = 0; u < 8; ++u) cs = fmaxf(cs, fmaxf(fmaxf(v[u].x, v[u].y), fmaxf(v[u].z, v[u].w)));
    }
  }
  float val[NC];
#pragma unroll
  for (int k = 0; k < NC; ++k) val[k] = 0.f;
  for (int p0 = 0; p0 < P; p0 += CB) {
    if (p0 > 0) load(p0);
#pragma unroll
    for (int b = 0; b < CB; ++b) {
      const int p = p0 + b;
      if (live && p < P) {
        const float c = cc[b];
        const float w = c == -INFINITY ? 0.f : exp2f(c - cf);
#pragma unroll
        for (int k = 0; k < NC; ++k) val[k] = fmaf(w, x[b][k], val[k]);
      }
    }
  }
  cs = warp_max(cs);
  if ((tid & 31) == 0) red[tid >> 5] = cs;
  __syncthreads();
  cs = red[0];
#pragma unroll
  for (int w = 1; w < kThreads / 32; ++w) cs = fmaxf(cs, red[w]);
  if (blockIdx.x == 0 && tid == 0) Sc[head] = cs;

  const float rel = cf > -INFINITY ? exp2f(cf - cs) : 0.f;  // the row relative to c*
  float amax = 0.f, den = 0.f;
#pragma unroll
  for (int k = 0; k < NC; ++k) {
    const int n = g + 8 * k;
    if (live && n < D1) S[(static_cast<size_t>(head) * m + f) * D1 + n] = val[k] * rel;
    if (n <= D) amax = fmaxf(amax, fabsf(val[k]));  // the normaliser must fit fp16 too
    if (n == D) den = val[k];
  }
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
  // amax = mant * 2^(ex + 15), mant in [0.5, 1), so amax * 2^-ex lies in [2^14, 2^15)
  int ex = 0;
  if (amax >= 1.17549435e-38f) {
    ex = ((__float_as_int(amax) >> 23) & 0xFF) - 126 - 15;
  } else if (amax > 0.f) {  // subnormal
    frexpf(amax, &ex);
    ex -= 15;
  }
  // 2^-ex as two normal factors (|ex| <= 164), an exact scaling wherever the result is normal
  const int ea = -ex / 2, eb = -ex - ea;
  const float sa = __int_as_float((127 + ea) << 23), sb = __int_as_float((127 + eb) << 23);
#pragma unroll
  for (int k = 0; k < NC; ++k) {
    const int n = g + 8 * k;
    if (n <= D) stage[n][fl] = __float2half_rn(val[k] * sa * sb);
  }
  stage[D + 1 + g][fl] = __float2half_rn(0.f);              // rows D+1 .. D+8
  if (g < 7) stage[D + 9 + g][fl] = __float2half_rn(0.f);  // rows D+9 .. D+15
  unsigned char* img = op + static_cast<size_t>(head) * op_bytes;
  // tail: the exponent of each feature, then its normaliser entry with the same scaling
  float* tail = reinterpret_cast<float*>(img + static_cast<size_t>(op_rows) * 128 * op_atoms);
  if (g == 0) tail[f] = live && cf > -INFINITY ? static_cast<float>(ex) + (cf - cs) : -INFINITY;
  if ((D & 7) == g) tail[op_tail + f] = live ? den * sa * sb : 0.f;
  __syncthreads();
  // the image holds 64 features per 128-byte row (dimension n), 16-byte chunk c at c ^ (n % 8):
  // this CTA's 32 features are four chunks of each row of its 64-feature atom
  const int atom = f0 >> 6;
  if (atom < op_atoms)
    for (int i = tid; i < op_rows * 4; i += kThreads) {
      const int n = i >> 2, c4 = i & 3, chunk = ((f0 & 63) >> 3) + c4;
      const size_t off = static_cast<size_t>(atom) * op_rows * 128 + static_cast<size_t>(n) * 128 + ((chunk ^ (n & 7)) << 4);
      *reinterpret_cast<uint4*>(img + off) = *reinterpret_cast<const uint4*>(&stage[n][8 * c4]);
    }
}

// grid (ceil(L/32), B*H), 256 threads.
// W row f of kv head g at W + g * w_head + f * w_row (w_head = 0, w_row = D: one W for all heads).
template <typename T, int D, int FMAP>
__global__ void __launch_bounds__(kThreads) query_pass_kernel(
    const T* __restrict__ Q, const float* __restrict__ W, const float* __restrict__ S,
    T* __restrict__ out, int L, int m, int H, int Hkv, float wscale, long w_head, int w_row) {
  constexpr int D1 = D + 1;
  constexpr int NE = (kQT * D1 + kThreads - 1) / kThreads;
  extern __shared__ float smem[];
  const int mp = m + 1;
  float* Qs = smem;               // [kQT][D1]
  float* Ws = Qs + kQT * D1;      // [kFB][D1]
  float* O = Ws + kFB * D1;       // [kQT][D1 + 1]
  float* U = O + kQT * (D1 + 1);  // [kQT][m + 1]

  const int tid = threadIdx.x;
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int kvh = b * Hkv + h / (H / Hkv);
  const int q0 = blockIdx.x * kQT, qw = min(kQT, L - q0);
  const T* Qh = Q + static_cast<size_t>(bh) * L * D;
  const float* Sh = S + static_cast<size_t>(kvh) * m * D1;
  const float* Wh = W + kvh * w_head;

  for (int i = tid; i < kQT * D; i += kThreads) {
    const int r = i / D, j = i % D;
    Qs[r * D1 + j] = r < qw ? to_f32(Qh[static_cast<size_t>(q0 + r) * D + j]) : 0.f;
  }
  for (int f0 = 0; f0 < m; f0 += kFB) {
    const int fbw = min(kFB, m - f0);
    __syncthreads();  // Qs ready / previous block done with Ws
    for (int i = tid; i < kFB * D; i += kThreads) {
      const int f = i / D, j = i % D;
      Ws[f * D1 + j] = f < fbw ? Wh[static_cast<size_t>(f0 + f) * w_row + j] * wscale : 0.f;
    }
    __syncthreads();
    for (int i = tid; i < kQT * kFB; i += kThreads) {
      const int r = i / kFB, f = i % kFB;
      if (f < fbw) {
        float s = 0.f;
#pragma unroll 16
        for (int j = 0; j < D; ++j) s = fmaf(Qs[r * D1 + j], Ws[f * D1 + j], s);
        U[r * mp + f0 + f] = s;
      }
    }
  }
  __syncthreads();
  {  // per-row max over the m features, then phi in place; 8 threads per row
    const int r = tid >> 3, k = tid & 7;
    if (FMAP == kExp) {
      float mx = -INFINITY;
      for (int f = k; f < m; f += 8) mx = fmaxf(mx, U[r * mp + f]);
#pragma unroll
      for (int o = 4; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      for (int f = k; f < m; f += 8) U[r * mp + f] = exp2f(U[r * mp + f] - mx);
    } else {
      for (int f = k; f < m; f += 8) U[r * mp + f] = fmaxf(U[r * mp + f], 0.f);
    }
  }
  float acc[NE];
#pragma unroll
  for (int k = 0; k < NE; ++k) acc[k] = 0.f;
  // out rows += phi S, 64 state rows at a time staged in shared memory (in place of W'), the
  // features summed in order f = 0 .. m - 1
  for (int f0 = 0; f0 < m; f0 += kFB) {
    const int fbw = min(kFB, m - f0);
    __syncthreads();  // phi is in place / the previous rows are used
    for (int i = tid; i < fbw * D1; i += kThreads) Ws[i] = Sh[static_cast<size_t>(f0) * D1 + i];
    __syncthreads();
    for (int f = 0; f < fbw; ++f) {
#pragma unroll
      for (int k = 0; k < NE; ++k) {
        const int e = tid + k * kThreads;
        if (e < kQT * D1) {
          const int r = e / D1, c = e % D1;
          acc[k] = fmaf(U[r * mp + f0 + f], Ws[f * D1 + c], acc[k]);
        }
      }
    }
  }
#pragma unroll
  for (int k = 0; k < NE; ++k) {
    const int e = tid + k * kThreads;
    if (e < kQT * D1) O[(e / D1) * (D1 + 1) + e % D1] = acc[k];
  }
  __syncthreads();
  T* Oh = out + static_cast<size_t>(bh) * L * D;
  for (int i = tid; i < kQT * D; i += kThreads) {
    const int r = i / D, c = i % D;
    if (r < qw) store_as(&Oh[static_cast<size_t>(q0 + r) * D + c], O[r * (D1 + 1) + c] / O[r * (D1 + 1) + D]);
  }
}

// Linformer notes page, "4 Model": the projections E K and F V (k x d per kv head) of the keys
// and values along the sequence.  grid (P, B*Hkv, ceil(k/64)), 256 threads: the CTA sums its
// chunk of tokens for 64 projected rows into the key pass's partial-state layout, F V (with the
// constant column 1 on chunk 0 only, so that the reduction's sum is 1) as head h and
// kscale E K as head heads + h, every stabiliser 0.  Thread (ty, tx) owns rows 4 ty .. 4 ty + 3
// and columns tx, tx + 16, ... of both products.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) linformer_proj_kernel(
    const T* __restrict__ K, const T* __restrict__ V, const float* __restrict__ E, const float* __restrict__ F,
    float* __restrict__ part_S, float* __restrict__ part_c, int L, int kp, int P, int chunk, int nsb, int heads,
    float kscale) {
  constexpr int D1 = D + 1;
  constexpr int CT = D / 16;
  constexpr int TT = 32;
  extern __shared__ float smem[];
  float* Es = smem;             // [64][TT + 1]
  float* Fs = Es + 64 * (TT + 1);  // [64][TT + 1]
  float* Ks = Fs + 64 * (TT + 1);  // [TT][D1]
  float* Vs = Ks + TT * D1;        // [TT][D1]
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int p = blockIdx.x, head = blockIdx.y, j0 = blockIdx.z * 64;
  const int t_begin = p * chunk, t_end = min(L, t_begin + chunk);
  const T* Kh = K + static_cast<size_t>(head) * L * D;
  const T* Vh = V + static_cast<size_t>(head) * L * D;
  float ak[4][CT], av[4][CT];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int c = 0; c < CT; ++c) ak[i][c] = av[i][c] = 0.f;
  for (int t0 = t_begin; t0 < t_end; t0 += TT) {
    const int tw = min(TT, t_end - t0);
    __syncthreads();  // the previous step is done with the tiles
    for (int i = tid; i < 64 * TT; i += kThreads) {
      const int j = i / TT, t = i % TT;
      const bool ok = j0 + j < kp && t < tw;
      Es[j * (TT + 1) + t] = ok ? E[static_cast<size_t>(j0 + j) * L + t0 + t] : 0.f;
      Fs[j * (TT + 1) + t] = ok ? F[static_cast<size_t>(j0 + j) * L + t0 + t] : 0.f;
    }
    for (int i = tid; i < TT * D; i += kThreads) {
      const int t = i / D, c = i % D;
      Ks[t * D1 + c] = t < tw ? to_f32(Kh[static_cast<size_t>(t0 + t) * D + c]) : 0.f;
      Vs[t * D1 + c] = t < tw ? to_f32(Vh[static_cast<size_t>(t0 + t) * D + c]) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int t = 0; t < TT; ++t) {
      float e[4], f[4], kv[CT], vv[CT];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        e[i] = Es[(4 * ty + i) * (TT + 1) + t];
        f[i] = Fs[(4 * ty + i) * (TT + 1) + t];
      }
#pragma unroll
      for (int c = 0; c < CT; ++c) {
        kv[c] = Ks[t * D1 + tx + 16 * c];
        vv[c] = Vs[t * D1 + tx + 16 * c];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < CT; ++c) {
          ak[i][c] = fmaf(e[i], kv[c], ak[i][c]);
          av[i][c] = fmaf(f[i], vv[c], av[i][c]);
        }
    }
  }
  float* outV = part_S + (static_cast<size_t>(head) * P + p) * static_cast<size_t>(kp) * D1;
  float* outK = part_S + (static_cast<size_t>(heads + head) * P + p) * static_cast<size_t>(kp) * D1;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int j = j0 + 4 * ty + i;
    if (j >= kp) continue;
#pragma unroll
    for (int c = 0; c < CT; ++c) {
      outK[static_cast<size_t>(j) * D1 + tx + 16 * c] = ak[i][c] * kscale;
      outV[static_cast<size_t>(j) * D1 + tx + 16 * c] = av[i][c];
    }
    if (tx == 0) {
      outK[static_cast<size_t>(j) * D1 + D] = 0.f;
      outV[static_cast<size_t>(j) * D1 + D] = p == 0 ? 1.f : 0.f;
      part_c[(static_cast<size_t>(head) * P + p) * nsb + j] = 0.f;
      part_c[(static_cast<size_t>(heads + head) * P + p) * nsb + j] = 0.f;
    }
  }
}

template <typename T, int D>
int launch_linformer_proj(const void* K, const void* V, const float* E, const float* F, void* partials,
                          const Plan& pk, int heads, cudaStream_t st) {
  constexpr int D1 = D + 1;
  const size_t smem = sizeof(float) * (2 * 64 * 33 + 2 * 32 * D1);
  auto kern = linformer_proj_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "projection attribute: %s", cudaGetErrorString(e));
  dim3 grid(pk.P, heads, (pk.m + 63) / 64);
  char* base = static_cast<char*>(partials);
  const float kscale = static_cast<float>(std::pow(static_cast<double>(D), -0.25));
  kern<<<grid, kThreads, smem, st>>>(static_cast<const T*>(K), static_cast<const T*>(V), E, F,
                                     reinterpret_cast<float*>(base + pk.part_S_off),
                                     reinterpret_cast<float*>(base + pk.part_c_off), pk.L, pk.m, pk.P, pk.chunk,
                                     pk.nsb, heads, kscale);
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "projection launch: %s", cudaGetErrorString(e));
  return FAVOR_OK;
}

// softmax(Q Kp^T / sqrt(d)) Vp with the state S (head h: [F V | 1], head heads + h: d^-1/4 E K):
// the query pass with the exp map, reading kv head h's projected keys as its W (row stride d + 1).
template <typename T, int D>
int launch_linformer_query(const void* Q, const void* state, void* out, const Plan& pq, const Plan& pk,
                           cudaStream_t st) {
  constexpr int D1 = D + 1;
  const size_t smem = sizeof(float) * (kQT * D1 + kFB * D1 + kQT * (D1 + 1) + kQT * (pq.m + 1));
  auto kern = query_pass_kernel<T, D, kExp>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "projected query attribute: %s", cudaGetErrorString(e));
  dim3 grid((pq.L + kQT - 1) / kQT, pq.B * pq.H);
  const float* S = reinterpret_cast<const float*>(static_cast<const char*>(state) + pk.st_S_off);
  const int heads = pq.B * pq.Hkv;
  const float* Wk = S + static_cast<size_t>(heads) * pq.m * D1;
  kern<<<grid, kThreads, smem, st>>>(static_cast<const T*>(Q), Wk, S, static_cast<T*>(out), pq.L, pq.m, pq.H, pq.Hkv,
                                     pq.wscale, static_cast<long>(pq.m) * D1, D1);
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "projected query launch: %s", cudaGetErrorString(e));
  return FAVOR_OK;
}


template <typename T, int D, int FMAP = kExp>
int launch_key(const void* K, const void* V, const float* W, void* partials, const Plan& p,
               cudaStream_t st) {
  constexpr int D1 = D + 1;
  const size_t smem = sizeof(float) * (kFB * D1 + 2 * kTT * D1 + kTT * (kFB + 1) + kThreads / 32);
  auto kern = key_pass_kernel<T, D, FMAP>;
  const float wscale = FMAP == kExp ? p.wscale : relu_wscale(p.d);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "key pass attribute: %s", cudaGetErrorString(e));
  dim3 grid(p.P, p.B * p.Hkv, (p.m + kFB - 1) / kFB);
  char* base = static_cast<char*>(partials);
  kern<<<grid, kThreads, smem, st>>>(static_cast<const T*>(K), static_cast<const T*>(V), W,
                                     reinterpret_cast<float*>(base + p.part_S_off),
                                     reinterpret_cast<float*>(base + p.part_c_off), p.L, p.m, p.P,
                                     p.chunk, p.nsb, wscale, p.nscale);
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "key pass launch: %s", cudaGetErrorString(e));
  return FAVOR_OK;
}

template <typename T, int D, int FMAP = kExp>
int launch_query(const void* Q, const float* W, const void* state, void* out, const Plan& p,
                 cudaStream_t st) {
  constexpr int D1 = D + 1;
  const size_t smem = sizeof(float) * (kQT * D1 + kFB * D1 + kQT * (D1 + 1) + kQT * (p.m + 1));
  auto kern = query_pass_kernel<T, D, FMAP>;
  const float wscale = FMAP == kExp ? p.wscale : relu_wscale(p.d);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "query pass attribute: %s", cudaGetErrorString(e));
  dim3 grid((p.L + kQT - 1) / kQT, p.B * p.H);
  const char* base = static_cast<const char*>(state);
  kern<<<grid, kThreads, smem, st>>>(static_cast<const T*>(Q), W,
                                     reinterpret_cast<const float*>(base + p.st_S_off),
                                     static_cast<T*>(out), p.L, p.m, p.H, p.Hkv, wscale, 0L, D);
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "query pass launch: %s", cudaGetErrorString(e));
  return FAVOR_OK;
}

}  // namespace

int simt_key_pass(int dtype, const void* K, const void* V, const float* W, void* partials,
                  const Plan& p, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == FAVOR_F32)
    return p.d == 64 ? launch_key<float, 64>(K, V, W, partials, p, st) : launch_key<float, 128>(K, V, W, partials, p, st);
  return p.d == 64 ? launch_key<__nv_bfloat16, 64>(K, V, W, partials, p, st)
                   : launch_key<__nv_bfloat16, 128>(K, V, W, partials, p, st);
}

int simt_state_reduce(const void* partials, void* state, const Plan& p, void* stream, bool overlap) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  dim3 grid(p.op_tail / 32, p.B * p.Hkv);
  const char* pb = static_cast<const char*>(partials);
  char* sb = static_cast<char*>(state);
  auto kern = p.d == 64 ? state_reduce_kernel<64> : state_reduce_kernel<128>;
  cudaError_t e = launch_overlapped(
      kern, grid, dim3(kThreads), 0, st, overlap, reinterpret_cast<const float*>(pb + p.part_S_off),
      reinterpret_cast<const float*>(pb + p.part_c_off), reinterpret_cast<float*>(sb + p.st_S_off),
      reinterpret_cast<float*>(sb + p.st_c_off), reinterpret_cast<unsigned char*>(sb + p.st_op_off), p.P, p.m, p.nsb,
      p.op_atoms, p.op_tail, p.op_bytes, p.op_rows);
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "state reduce launch: %s", cudaGetErrorString(e));
  return FAVOR_OK;
}

int simt_key_pass_relu(int dtype, const void* K, const void* V, const float* W, void* partials, const Plan& p,
                       void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == FAVOR_F32)
    return p.d == 64 ? launch_key<float, 64, kRelu>(K, V, W, partials, p, st)
                     : launch_key<float, 128, kRelu>(K, V, W, partials, p, st);
  return p.d == 64 ? launch_key<__nv_bfloat16, 64, kRelu>(K, V, W, partials, p, st)
                   : launch_key<__nv_bfloat16, 128, kRelu>(K, V, W, partials, p, st);
}

int simt_query_pass_relu(int dtype, const void* Q, const float* W, const void* state, void* out, const Plan& p,
                         void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == FAVOR_F32)
    return p.d == 64 ? launch_query<float, 64, kRelu>(Q, W, state, out, p, st)
                     : launch_query<float, 128, kRelu>(Q, W, state, out, p, st);
  return p.d == 64 ? launch_query<__nv_bfloat16, 64, kRelu>(Q, W, state, out, p, st)
                   : launch_query<__nv_bfloat16, 128, kRelu>(Q, W, state, out, p, st);
}

int simt_linformer_proj(int dtype, const void* K, const void* V, const float* E, const float* F, void* partials,
                        const Plan& pk, int heads, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == FAVOR_F32)
    return pk.d == 64 ? launch_linformer_proj<float, 64>(K, V, E, F, partials, pk, heads, st)
                      : launch_linformer_proj<float, 128>(K, V, E, F, partials, pk, heads, st);
  return pk.d == 64 ? launch_linformer_proj<__nv_bfloat16, 64>(K, V, E, F, partials, pk, heads, st)
                    : launch_linformer_proj<__nv_bfloat16, 128>(K, V, E, F, partials, pk, heads, st);
}

int simt_linformer_query(int dtype, const void* Q, const void* state, void* out, const Plan& pq, const Plan& pk,
                         void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == FAVOR_F32)
    return pq.d == 64 ? launch_linformer_query<float, 64>(Q, state, out, pq, pk, st)
                      : launch_linformer_query<float, 128>(Q, state, out, pq, pk, st);
  return pq.d == 64 ? launch_linformer_query<__nv_bfloat16, 64>(Q, state, out, pq, pk, st)
                    : launch_linformer_query<__nv_bfloat16, 128>(Q, state, out, pq, pk, st);
}

int simt_query_pass(int dtype, const void* Q, const float* W, const void* state, void* out,
                    const Plan& p, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == FAVOR_F32)
    return p.d == 64 ? launch_query<float, 64>(Q, W, state, out, p, st) : launch_query<float, 128>(Q, W, state, out, p, st);
  return p.d == 64 ? launch_query<__nv_bfloat16, 64>(Q, W, state, out, p, st)
                   : launch_query<__nv_bfloat16, 128>(Q, W, state, out, p, st);
}

}  // namespace favor
