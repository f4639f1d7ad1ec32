// FAVOR+ incremental decoding against a cached per-kv-head state (sm_100a, CUDA cores).
//
// "Fast Transformer Decoding: One Write-Head is All You Need" (研究动机与目标 / motivation;
// 提出的方法 / proposed method): in incremental decoding every step reads the whole key/value
// cache, so memory bandwidth bounds it, and H query heads sharing one key/value head shrink
// that cache.  With FAVOR+ ("Rethinking Attention with Performers", Abstract: linear space)
// the cache of each kv head is its fixed-size state, m x (d + 1) plus one stabiliser per feature,
// whatever the number of tokens seen:
//   state     S[f, :] = sum_t 2^(a_t,f - c_f) [v_t | 1],  a_t,f = W'_f . k_t - n(k_t)  (log2 units)
//   update    a new key: c_f' = max(c_f, a_f); S[f, :] = 2^(c_f - c_f') S[f, :] + 2^(a_f - c_f') [v | 1]
//   query     e_f = W'_f . q + c_f;  out = sum_f 2^(e_f - M) S[f, :d] / sum_f 2^(e_f - M) S[f, d]
// with M = max_f e_f (the query's stabiliser; -|q'|^2/2 and 1/sqrt(m) cancel in the ratio).
// The update keeps the exact running maximum, so it is exact in fp32 up to rounding.
//
// One thread-block cluster of 8 CTAs per kv head; CTA r of a cluster owns features
// [r m/8, (r + 1) m/8): it updates those rows of the state and computes, for each of the G query
// heads, its maximum exponent and the partial sums of its rows.  The partials are combined across
// the cluster through distributed shared memory: CTA r finishes the query heads g = r, r + 8, ...
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "favor_internal.h"
#include "launch.cuh"
#include "sm100_ptx.cuh"

namespace cg = cooperative_groups;

namespace favor {
namespace {

using sm100::ex2;

constexpr int kCluster = 8;
constexpr int kThreads = 256;
constexpr int kMaxG = 64;

__device__ __forceinline__ void store_as(float* p, float x) { *p = x; }
__device__ __forceinline__ void store_as(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// Shared-memory layout of one CTA (offsets in floats; the float4 regions start on 16 bytes).
struct DecodeSmem {
  int D, G, FPC, PS;
  int x, v, wl, sl, cl, snew, fac, a, eq, phi, part, total;
  __host__ __device__ static int round4(int n) { return (n + 3) & ~3; }
  __host__ __device__ DecodeSmem(int D_, int G_, int FPC_) : D(D_), G(G_), FPC(FPC_) {
    PS = (G + 7) / 8 * 8 + 4;            // phi row stride: whole groups of 8 query heads, plus 4 against bank conflicts
    x = 0;                               // [1 + G][D]: the key, then the G queries
    v = x + (1 + G) * D;                 // [D]: the value
    wl = v + D;                          // [FPC][D]: this CTA's rows of W
    sl = wl + FPC * D;                   // [FPC][D + 1]: its state rows, as stored
    cl = sl + round4(FPC * (D + 1));     // [FPC]: the stabilisers c
    snew = cl + round4(FPC);             // [FPC][D]: the updated rows S'[f, :D]
    fac = snew + FPC * D;                // [FPC][4]: 2^(c - c'), 2^(a - c'), c', S'[f, D]
    a = fac + 4 * FPC;                   // [FPC]: the new key's exponents a = W'k - n(k)
    eq = a + FPC;                        // [G][FPC]: W'q_g
    phi = round4(eq + G * FPC);          // [FPC][PS]: 2^(e_gf - M_g), zero for g >= G
    part = phi + FPC * PS;               // [G][D + 4]: the D numerator sums, the normaliser sum, M_g
    total = part + G * (D + 4);
    // bf16 k, q and v land first in [snew, total) (unused until the dots), which always holds (2 + G) D
    // of them: FPC D + G (D + 4) >= 2 D + G D floats
  }
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async4(float* dst, const float* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async16(float* dst, const float* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// Cluster barrier halves: arrive with release (this thread's earlier shared-memory writes become visible
// to the cluster) or relaxed (nothing to publish), and wait with acquire.
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

__device__ __forceinline__ float dot4(float4 w, float4 x, float acc) {
  return fmaf(w.w, x.w, fmaf(w.z, x.z, fmaf(w.y, x.y, fmaf(w.x, x.x, acc))));
}

template <typename T, int D>
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads) decode_step_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, const float* __restrict__ W,
    float* __restrict__ state, T* __restrict__ out, int G, int m, float wscale, float nscale) {
  constexpr int NGQ = kThreads / D;  // threads per state column in the sums and the combine
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(16) float sm[];
  const int FPC = m / kCluster;
  const DecodeSmem L(D, G, FPC);
  const int GP = L.PS - 4;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = static_cast<int>(cluster.block_rank());
  const int kvh = blockIdx.x / kCluster;
  const int f0 = r * FPC;
  float* Sg = state + static_cast<size_t>(kvh) * m * (D + 2);  // S [m][D + 1], then c [m]
  float* cg_ = Sg + static_cast<size_t>(m) * (D + 1);

  // Nothing is read or written before the kernels ahead of this one on the stream have completed;
  // the next step may be scheduled at once and waits in the same place.
  griddep_wait();
  griddep_launch_dependents();

  // 1. one burst of asynchronous copies: this CTA's rows of W, of the state and their stabilisers, and the
  //    new key, queries and value (bf16 widened to fp32 once they have landed)
  for (int c = tid; c < FPC * (D / 4); c += kThreads) {
    const int f = c / (D / 4), j = 4 * (c - f * (D / 4));
    cp_async16(&sm[L.wl + f * D + j], W + static_cast<size_t>(f0 + f) * D + j);
  }
  const float* Ssrc = Sg + static_cast<size_t>(f0) * (D + 1);
  for (int i = tid; i < FPC * (D + 1); i += kThreads) cp_async4(&sm[L.sl + i], Ssrc + i);
  for (int i = tid; i < FPC; i += kThreads) cp_async4(&sm[L.cl + i], cg_ + f0 + i);
  {  // k, the G queries and v in that order ([k | q | v] is also the fp32 layout of x and v)
    constexpr int E = 16 / sizeof(T);  // elements per 16-byte copy
    const int nk = D / E, nq = G * D / E;
    T* stage = sizeof(T) == 4 ? reinterpret_cast<T*>(&sm[L.x]) : reinterpret_cast<T*>(&sm[L.snew]);
    for (int c = tid; c < 2 * nk + nq; c += kThreads) {
      const T* src = c < nk        ? k + static_cast<size_t>(kvh) * D + c * E
                     : c < nk + nq ? q + static_cast<size_t>(kvh) * G * D + (c - nk) * E
                                   : v + static_cast<size_t>(kvh) * D + (c - nk - nq) * E;
      cp_async16(reinterpret_cast<float*>(stage + c * E), reinterpret_cast<const float*>(src));
    }
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  cp_async_wait_all();
  __syncthreads();
  if constexpr (sizeof(T) == 2) {  // widen the staged bf16 to fp32
    const __nv_bfloat162* st2 = reinterpret_cast<const __nv_bfloat162*>(&sm[L.snew]);
    for (int i = tid; i < (2 + G) * D / 2; i += kThreads)
      *reinterpret_cast<float2*>(&sm[L.x + 2 * i]) = __bfloat1622float2(st2[i]);
    __syncthreads();
  }

  // 2. the dots with W' = d^-1/4 log2(e) W: W'_f . q_g and a_f = W'_f . k - n(k), n(k) = d^-1/2 log2(e) |k|^2 / 2.
  //    Each lane keeps a 16-float slice (the float4s s, s + S, s + 2 S, s + 3 S) of four consecutive query rows
  //    and of the key in registers and streams W's rows past them; the S lanes of a row block add their
  //    slices by shuffles.  The warps split the row blocks into NRG groups, each group's warps the features;
  //    the first group's warps also take the key.
  {
    constexpr int S = D / 16, RB = 32 / S;  // lanes per row block, row blocks per warp
    const int JBq = (G + 3) / 4, NRG = (JBq + RB - 1) / RB, NFP = (kThreads / 32) / NRG;
    const int rg = warp % NRG, fp = warp / NRG;
    if (fp < NFP) {
      const int s = lane % S, jb = rg * RB + lane / S;
      float4 xr[4][4], kr[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float4* x4 = reinterpret_cast<const float4*>(&sm[L.x + (1 + min(4 * jb + u, G - 1)) * D]);
#pragma unroll
        for (int t = 0; t < 4; ++t) xr[u][t] = x4[s + S * t];
      }
      float nk = 0.f;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        kr[t] = reinterpret_cast<const float4*>(&sm[L.x])[s + S * t];
        nk = dot4(kr[t], kr[t], nk);
      }
#pragma unroll
      for (int o = S / 2; o > 0; o >>= 1) nk += __shfl_xor_sync(0xffffffffu, nk, o);
      for (int f = fp; f < FPC; f += NFP) {
        const float4* w4 = reinterpret_cast<const float4*>(&sm[L.wl + f * D]);
        float4 w[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) w[t] = w4[s + S * t];
        float acc[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
#pragma unroll
          for (int u = 0; u < 4; ++u) acc[u] = dot4(w[t], xr[u][t], acc[u]);
          if (rg == 0) acc[4] = dot4(w[t], kr[t], acc[4]);
        }
#pragma unroll
        for (int o = S / 2; o > 0; o >>= 1)
#pragma unroll
          for (int u = 0; u < 5; ++u) acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], o);
        if (s == 0) {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (4 * jb + u < G) sm[L.eq + (4 * jb + u) * FPC + f] = acc[u] * wscale;
        }
        if (rg == 0 && lane == 0) sm[L.a + f] = acc[4] * wscale - nk * nscale;
      }
    }
  }
  __syncthreads();

  // 3. per feature (lanes; at most two features each): c' = max(c, a), 2^(c - c'), 2^(a - c') and
  //    the updated normaliser entry S'[f, D]; per query head (two per warp at a time): e_gf = W'q_g + c'_f,
  //    M_g = max_f e_gf, 2^(e_gf - M_g) and the normaliser sum sum_f 2^(e_gf - M_g) S'[f, D]
  {
    float cn[2], sden[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int f = lane + 32 * u;
      cn[u] = 0.f;
      sden[u] = 0.f;
      if (f < FPC) {
        const float a = sm[L.a + f], c = sm[L.cl + f];
        cn[u] = fmaxf(c, a);
        const float sc = c == -INFINITY ? 0.f : ex2(c - cn[u]), wn = ex2(a - cn[u]);
        sden[u] = fmaf(sm[L.sl + f * (D + 1) + D], sc, wn);
        if (warp == 0) *reinterpret_cast<float4*>(&sm[L.fac + 4 * f]) = make_float4(sc, wn, cn[u], sden[u]);
      }
    }
    for (int g = warp; g < GP; g += 16) {
      const int gg[2] = {g, g + 8};  // g + 8 < GP exactly when it is a head (or padding) of this group
      float e[2][2], M[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int f = lane + 32 * u;
          e[h][u] = gg[h] < G && f < FPC ? sm[L.eq + gg[h] * FPC + f] + cn[u] : -INFINITY;
          M[h] = fmaxf(M[h], e[h][u]);
        }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        M[0] = fmaxf(M[0], __shfl_xor_sync(0xffffffffu, M[0], o));
        M[1] = fmaxf(M[1], __shfl_xor_sync(0xffffffffu, M[1], o));
      }
      float den[2] = {0.f, 0.f};
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int f = lane + 32 * u;
          if (f < FPC && gg[h] < GP) {
            const float ph = gg[h] < G ? ex2(e[h][u] - M[h]) : 0.f;  // padding heads: zero weights
            sm[L.phi + f * L.PS + gg[h]] = ph;
            den[h] = fmaf(ph, sden[u], den[h]);
          }
        }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        den[0] += __shfl_xor_sync(0xffffffffu, den[0], o);
        den[1] += __shfl_xor_sync(0xffffffffu, den[1], o);
      }
      if (lane == 0) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
          if (gg[h] < G) {
            sm[L.part + gg[h] * (D + 4) + D] = den[h];
            sm[L.part + gg[h] * (D + 4) + D + 1] = M[h];
          }
      }
    }
  }
  __syncthreads();

  // 4. (a) the rank-one update S'[f, n] = 2^(c - c') S[f, n] + 2^(a - c') v[n], kept in shared memory
  for (int i = tid; i < FPC * D; i += kThreads) {
    const int f = i / D, n = i % D;
    const float2 sw = *reinterpret_cast<const float2*>(&sm[L.fac + 4 * f]);
    sm[L.snew + i] = fmaf(sm[L.sl + f * (D + 1) + n], sw.x, sw.y * sm[L.v + n]);
  }
  __syncthreads();
  //    (b) the numerator sums num_g[n] = sum_f 2^(e_gf - M_g) S'[f, n], each thread a tile of four query
  //    heads by four columns
  for (int it = tid; it < (G + 3) / 4 * (D / 4); it += kThreads) {
    const int nb = it % (D / 4), gb = it / (D / 4);
    float4 acc[4] = {};
#pragma unroll 4
    for (int f = 0; f < FPC; ++f) {
      const float4 p = *reinterpret_cast<const float4*>(&sm[L.phi + f * L.PS + 4 * gb]);
      const float4 sv = *reinterpret_cast<const float4*>(&sm[L.snew + f * D + 4 * nb]);
      const float pu[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        acc[u].x = fmaf(pu[u], sv.x, acc[u].x);
        acc[u].y = fmaf(pu[u], sv.y, acc[u].y);
        acc[u].z = fmaf(pu[u], sv.z, acc[u].z);
        acc[u].w = fmaf(pu[u], sv.w, acc[u].w);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (4 * gb + u < G) *reinterpret_cast<float4*>(&sm[L.part + (4 * gb + u) * (D + 4) + 4 * nb]) = acc[u];
  }
  cluster_arrive_release();  // this CTA's partials are published to the cluster

  // 5. the updated rows go back to the state while the other CTAs finish
  for (int i = tid; i < FPC * D; i += kThreads) {
    const int f = i / D, n = i % D;
    Sg[static_cast<size_t>(f0 + f) * (D + 1) + n] = sm[L.snew + i];
  }
  for (int f = tid; f < FPC; f += kThreads) {
    const float4 fc = *reinterpret_cast<const float4*>(&sm[L.fac + 4 * f]);
    Sg[static_cast<size_t>(f0 + f) * (D + 1) + D] = fc.w;
    cg_[f0 + f] = fc.z;
  }
  cluster_wait();  // every CTA's partials are visible

  // 6. CTA r finishes query heads g = r, r + 8, ...: the 8 CTAs' partials rescaled to the largest maximum
  {
    const float* parts[kCluster];
#pragma unroll
    for (int i = 0; i < kCluster; ++i) parts[i] = cluster.map_shared_rank(&sm[L.part], i);
    const int n = tid % D;
    for (int g = r + kCluster * (tid / D); g < G; g += kCluster * NGQ) {
      float Mi[kCluster], nu[kCluster], de[kCluster], M = -INFINITY;
#pragma unroll
      for (int i = 0; i < kCluster; ++i) {
        const float* pp = parts[i] + g * (D + 4);
        nu[i] = pp[n];
        de[i] = pp[D];
        Mi[i] = pp[D + 1];
      }
#pragma unroll
      for (int i = 0; i < kCluster; ++i) M = fmaxf(M, Mi[i]);
      float num = 0.f, den = 0.f;
#pragma unroll
      for (int i = 0; i < kCluster; ++i) {
        const float sc = ex2(Mi[i] - M);
        num = fmaf(sc, nu[i], num);
        den = fmaf(sc, de[i], den);
      }
      store_as(&out[(static_cast<size_t>(kvh) * G + g) * D + n], num * (1.f / den));
    }
  }
  cluster_arrive_relaxed();  // this CTA reads no other CTA's shared memory any more
  cluster_wait();            // and leaves only when no other CTA reads its own
}

__global__ void decode_init_kernel(float* __restrict__ state, size_t heads, int m, int D) {
  const size_t per = static_cast<size_t>(m) * (D + 2);
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < heads * per;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t j = i % per;
    state[i] = j < static_cast<size_t>(m) * (D + 1) ? 0.f : -INFINITY;
  }
}

template <typename T, int D>
int launch_decode(const void* q, const void* k, const void* v, const float* W, void* state, void* out, int B,
                  int H, int Hkv, int m, cudaStream_t st) {
  const int G = H / Hkv;
  const DecodeSmem L(D, G, m / kCluster);
  const size_t smem = sizeof(float) * L.total;
  auto kern = decode_step_kernel<T, D>;
  // the largest dynamic shared memory any supported shape needs, set once per kernel so that later calls
  // (for instance inside a stream capture) make no attribute call
  static const cudaError_t attr = [&] {
    int most = 0;
    for (int g = 1; g <= kMaxG; ++g)
      for (int mm = 16; mm <= 512; mm += 16) most = std::max(most, DecodeSmem(D, g, mm / kCluster).total);
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(sizeof(float) * most));
  }();
  cudaError_t e = attr;
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "decode step attribute: %s", cudaGetErrorString(e));
  const float wscale = static_cast<float>(std::pow(static_cast<double>(D), -0.25) * kLog2e);
  const float nscale = static_cast<float>(std::pow(static_cast<double>(D), -0.5) * kLog2e * 0.5);
  // the kernel touches no memory before griddepcontrol.wait, so it may always be scheduled early
  e = launch_overlapped(kern, dim3(kCluster * B * Hkv), dim3(kThreads), smem, st, true, static_cast<const T*>(q),
                        static_cast<const T*>(k), static_cast<const T*>(v), W, static_cast<float*>(state),
                        static_cast<T*>(out), G, m, wscale, nscale);
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "decode step launch: %s", cudaGetErrorString(e));
  return FAVOR_OK;
}

int check_decode_shape(int B, int H, int Hkv, int d, int m) {
  if (B < 1 || H < 1 || Hkv < 1)
    return set_errorf(FAVOR_ERR_UNSUPPORTED, "B, H and Hkv must be >= 1 (got %d, %d, %d)", B, H, Hkv);
  if (H % Hkv != 0) return set_errorf(FAVOR_ERR_UNSUPPORTED, "H (%d) must be a multiple of Hkv (%d)", H, Hkv);
  if (H / Hkv > kMaxG) return set_errorf(FAVOR_ERR_UNSUPPORTED, "at most %d query heads per kv head (got %d)", kMaxG, H / Hkv);
  if (d != 64 && d != 128) return set_errorf(FAVOR_ERR_UNSUPPORTED, "d must be 64 or 128 (got %d)", d);
  if (m < 16 || m > 512 || m % 16 != 0)
    return set_errorf(FAVOR_ERR_UNSUPPORTED, "m must be a multiple of 16 in [16, 512] (got %d)", m);
  if (static_cast<long>(B) * Hkv * kCluster > 2147483647L) return set_error(FAVOR_ERR_UNSUPPORTED, "too many kv heads");
  return FAVOR_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace favor

using namespace favor;

extern "C" {

size_t favor_decode_state_bytes(int B, int Hkv, int d, int m) {
  if (check_decode_shape(B, Hkv, Hkv, d, m) != FAVOR_OK) return 0;
  return sizeof(float) * static_cast<size_t>(B) * Hkv * m * (d + 2);
}

int favor_decode_init(void* state, int B, int Hkv, int d, int m, favor_stream_t stream) {
  int rc = check_decode_shape(B, Hkv, Hkv, d, m);
  if (rc != FAVOR_OK) return rc;
  if (!state || !aligned16(state)) return set_error(FAVOR_ERR_INVALID, "favor_decode_init: null or misaligned state");
  const size_t total = static_cast<size_t>(B) * Hkv * m * (d + 2);
  const int blocks = static_cast<int>((total + 255) / 256 < 4096 ? (total + 255) / 256 : 4096);
  decode_init_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<float*>(state), static_cast<size_t>(B) * Hkv, m, d);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "favor_decode_init: %s", cudaGetErrorString(e));
  return FAVOR_OK;
}

int favor_decode_step(int dtype, const void* q, const void* k, const void* v, const float* W, void* state,
                      void* out, int B, int H, int Hkv, int d, int m, favor_stream_t stream) {
  if (dtype != FAVOR_BF16 && dtype != FAVOR_F32)
    return set_errorf(FAVOR_ERR_INVALID, "favor_decode_step: dtype must be 0 or 1, got %d", dtype);
  int rc = check_decode_shape(B, H, Hkv, d, m);
  if (rc != FAVOR_OK) return rc;
  for (const void* p : {q, k, v, static_cast<const void*>(W), static_cast<const void*>(state),
                        static_cast<const void*>(out)})
    if (!p || !aligned16(p)) return set_error(FAVOR_ERR_INVALID, "favor_decode_step: null or not 16-byte aligned pointer");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == FAVOR_BF16)
    return d == 64 ? launch_decode<__nv_bfloat16, 64>(q, k, v, W, state, out, B, H, Hkv, m, st)
                   : launch_decode<__nv_bfloat16, 128>(q, k, v, W, state, out, B, H, Hkv, m, st);
  return d == 64 ? launch_decode<float, 64>(q, k, v, W, state, out, B, H, Hkv, m, st)
                 : launch_decode<float, 128>(q, k, v, W, state, out, B, H, Hkv, m, st);
}

}  // extern "C"
