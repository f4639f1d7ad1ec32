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

#include <cmath>

#include "favor_internal.h"

namespace cg = cooperative_groups;

namespace favor {
namespace {

constexpr int kCluster = 8;
constexpr int kThreads = 256;
constexpr int kMaxG = 64;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void store_as(float* p, float x) { *p = x; }
__device__ __forceinline__ void store_as(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

struct DecodeSmem {
  int D, G, FPC;
  // offsets in floats
  int kq, v, wl, sl, e, part, a, cn, sc, wn, misc, total;
  __host__ __device__ DecodeSmem(int D_, int G_, int FPC_) : D(D_), G(G_), FPC(FPC_) {
    kq = 0;                              // [1 + G][D]: the key, then the G queries
    v = kq + (1 + G) * D;                // [D]
    wl = v + D;                          // [FPC][D + 1]: this CTA's rows of W'
    sl = wl + FPC * (D + 1);             // [FPC][D + 1]: its updated state rows
    e = sl + FPC * (D + 1);              // [G][FPC]: exponents, then 2^(e - M_g)
    part = e + G * FPC;                  // [G][D + 2]: M_g, then the partial sums (read by the cluster)
    a = part + G * (D + 2);              // [FPC]: the new key's exponents
    cn = a + FPC;                        // [FPC]: the new stabilisers
    sc = cn + FPC;                       // [FPC]: 2^(c - c')
    wn = sc + FPC;                       // [FPC]: 2^(a - c')
    misc = wn + FPC;                     // [4]: n(k)
    total = misc + 4;
  }
};

template <typename T, int D>
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads) decode_step_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, const float* __restrict__ W,
    float* __restrict__ state, T* __restrict__ out, int G, int m, float wscale, float nscale) {
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ float sm[];
  const int FPC = m / kCluster;
  const DecodeSmem L(D, G, FPC);
  const int tid = threadIdx.x;
  const int r = static_cast<int>(cluster.block_rank());
  const int kvh = blockIdx.x / kCluster;
  const int f0 = r * FPC;
  float* Sg = state + static_cast<size_t>(kvh) * m * (D + 2);  // S [m][D + 1], then c [m]
  float* cg_ = Sg + static_cast<size_t>(m) * (D + 1);

  // 1. the new key, value and queries, and this CTA's rows of W' = d^-1/4 log2(e) W
  for (int i = tid; i < D; i += kThreads) {
    sm[L.kq + i] = to_f32(k[static_cast<size_t>(kvh) * D + i]);
    sm[L.v + i] = to_f32(v[static_cast<size_t>(kvh) * D + i]);
  }
  for (int i = tid; i < G * D; i += kThreads)
    sm[L.kq + D + i] = to_f32(q[static_cast<size_t>(kvh) * G * D + i]);
  for (int i = tid; i < FPC * D; i += kThreads) {
    const int f = i / D, j = i - f * D;
    sm[L.wl + f * (D + 1) + j] = W[static_cast<size_t>(f0 + f) * D + j] * wscale;
  }
  __syncthreads();
  if (tid < 32) {  // n(k) = d^-1/2 log2(e) |k|^2 / 2
    float s2 = 0.f;
    for (int i = tid; i < D; i += 32) s2 = fmaf(sm[L.kq + i], sm[L.kq + i], s2);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
    if (tid == 0) sm[L.misc] = s2 * nscale;
  }
  __syncthreads();
  // 2. W'_f . k and W'_f . q_g for this CTA's features (consecutive threads: consecutive features)
  for (int p = tid; p < FPC * (1 + G); p += kThreads) {
    const int j = p / FPC, f = p - j * FPC;
    const float* wr = &sm[L.wl + f * (D + 1)];
    const float* x = &sm[L.kq + j * D];
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 8
    for (int i = 0; i < D; i += 2) {
      acc0 = fmaf(wr[i], x[i], acc0);
      acc1 = fmaf(wr[i + 1], x[i + 1], acc1);
    }
    const float dot = acc0 + acc1;
    if (j == 0) sm[L.a + f] = dot - sm[L.misc];
    else sm[L.e + (j - 1) * FPC + f] = dot;
  }
  __syncthreads();
  // 3. the update's per-feature factors: c' = max(c, a), 2^(c - c'), 2^(a - c')
  for (int f = tid; f < FPC; f += kThreads) {
    const float a = sm[L.a + f], c = cg_[f0 + f];
    const float cn = fmaxf(c, a);
    sm[L.cn + f] = cn;
    sm[L.sc + f] = c == -INFINITY ? 0.f : exp2f(c - cn);
    sm[L.wn + f] = exp2f(a - cn);
  }
  __syncthreads();
  // 4. the rank-one update of this CTA's rows (coalesced along each row)
  for (int p = tid; p < FPC * (D + 1); p += kThreads) {
    const int f = p / (D + 1), n = p - f * (D + 1);
    const size_t gi = static_cast<size_t>(f0 + f) * (D + 1) + n;
    const float s = fmaf(Sg[gi], sm[L.sc + f], sm[L.wn + f] * (n < D ? sm[L.v + n] : 1.f));
    Sg[gi] = s;
    sm[L.sl + f * (D + 1) + n] = s;
  }
  for (int f = tid; f < FPC; f += kThreads) cg_[f0 + f] = sm[L.cn + f];
  // 5. each query head's exponents e = W'q + c', its maximum over this CTA's features, 2^(e - M)
  for (int p = tid; p < G * FPC; p += kThreads) {
    const int f = p % FPC;
    sm[L.e + p] += sm[L.cn + f];
  }
  __syncthreads();
  for (int g = tid; g < G; g += kThreads) {
    float mx = -INFINITY;
    for (int f = 0; f < FPC; ++f) mx = fmaxf(mx, sm[L.e + g * FPC + f]);
    sm[L.part + g * (D + 2)] = mx;
  }
  __syncthreads();
  for (int p = tid; p < G * FPC; p += kThreads) {
    const int g = p / FPC;
    sm[L.e + p] = exp2f(sm[L.e + p] - sm[L.part + g * (D + 2)]);
  }
  __syncthreads();
  // 6. partial sums over this CTA's features: num_g[n] = sum_f 2^(e_gf - M_g) S[f, n]
  for (int p = tid; p < G * (D + 1); p += kThreads) {
    const int g = p / (D + 1), n = p - g * (D + 1);
    const float* ph = &sm[L.e + g * FPC];
    float acc = 0.f;
    for (int f = 0; f < FPC; ++f) acc = fmaf(ph[f], sm[L.sl + f * (D + 1) + n], acc);
    sm[L.part + g * (D + 2) + 1 + n] = acc;
  }
  cluster.sync();  // every CTA's partials are in its shared memory
  // 7. CTA r finishes query heads r, r + 8, ...: rescale the 8 partials to the largest maximum
  const float* parts[kCluster];
#pragma unroll
  for (int i = 0; i < kCluster; ++i) parts[i] = cluster.map_shared_rank(&sm[L.part], i);
  for (int g = r; g < G; g += kCluster) {
    float M = -INFINITY;
#pragma unroll
    for (int i = 0; i < kCluster; ++i) M = fmaxf(M, parts[i][g * (D + 2)]);
    float* red = &sm[L.sl];  // this CTA's state rows are no longer needed: [D + 1] sums
    for (int n = tid; n <= D; n += kThreads) {
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < kCluster; ++i) {
        const float Mi = parts[i][g * (D + 2)];
        if (Mi > -INFINITY) acc = fmaf(exp2f(Mi - M), parts[i][g * (D + 2) + 1 + n], acc);
      }
      red[n] = acc;
    }
    __syncthreads();
    const float inv = 1.f / red[D];
    T* o = out + (static_cast<size_t>(kvh) * G + g) * D;
    for (int n = tid; n < D; n += kThreads) store_as(&o[n], red[n] * inv);
    __syncthreads();
  }
  cluster.sync();  // no CTA leaves while another still reads its shared memory
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
  // the largest dynamic shared memory any shape needs (G = 64, m = 512), set once per kernel so that
  // later calls (for instance inside a stream capture) make no attribute call
  static const cudaError_t attr = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
      static_cast<int>(sizeof(float) * DecodeSmem(D, kMaxG, 512 / kCluster).total));
  cudaError_t e = attr;
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "decode step attribute: %s", cudaGetErrorString(e));
  const float wscale = static_cast<float>(std::pow(static_cast<double>(D), -0.25) * kLog2e);
  const float nscale = static_cast<float>(std::pow(static_cast<double>(D), -0.5) * kLog2e * 0.5);
  kern<<<dim3(kCluster * B * Hkv), dim3(kThreads), smem, st>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), W, static_cast<float*>(state),
      static_cast<T*>(out), G, m, wscale, nscale);
  e = cudaGetLastError();
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
