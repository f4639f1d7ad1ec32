// FAVOR+ on the sm_100a tensor cores (tcgen05 + TMEM + TMA), bf16 inputs.
//
// "Rethinking Attention with Performers" (Abstract; 제안 방법 / proposed
// method): out = phi(Q')(phi(K')^T [V|1]) / last column, with positive random
// features phi(x') = exp(W x' - |x'|^2/2)/sqrt(m).  Both contractions on each
// side are dense, so they run on the tensor cores; the exp feature map (m
// exponentials per token) runs on the MUFU between them.  Everything is in log2
// units: W' = d^-1/4 log2(e) W, n(k) = d^-1/2 log2(e) |k|^2 / 2.
//
// Key pass, d = 64 (one CTA per 128-feature group x key chunk x kv head; two
// epilogue warpgroups on alternate 128-token tiles, each with its own MMA issuer):
//   MMA1  U^T[f, t] = (W'hi + W'lo)[f, :] . K[t, :]   A = W' halves (smem), B = K tile (TMA)
//   exp   phi^T[f, t] = 2^(U^T - n(k_t) - c_f)        bf16, into its own TMEM buffer
//   MMA2  S[f, :] += phi^T[f, :] . V                  A = phi^T (TMEM), B = V tile (MN-major)
// so every epilogue thread owns one feature (TMEM lane) and reads its U^T row once.
// c_f is the feature's running max exponent, raised only when a tile exceeds it by
// more than 2^8 (S and the normaliser sum are then rescaled exactly); the state
// reduction brings all chunks to one constant per feature.
// Key pass, d = 128: the lock-step variant (both warpgroups on each tile, W' hi + lo
// in TMEM as the A operand, one N = d + 16 MMA2 against [V | ones]).
//
// Query pass (one persistent CTA per SM over a contiguous range of 128-query tiles;
// two epilogue warpgroups on alternate tiles, each with its own MMA issuer):
//   MMA1  U[q, f] = (2^-k_q Q)[q, :] . W'[f, :]       fp16, per block of FB features
//   exp   phi'[q, f] = 2^(2^k_q U + e_f - c_q)         fp16, into its own TMEM buffer;
//                                                       c_q = the row max, raised lazily
//   MMA2  O[q, :] += phi'[q, block] . S'[block, :]      A = phi' (TMEM), B = fp16 state image
//   out = O / (phi' . s) -> bf16 -> TMA store.
// The state image holds each feature row scaled by its own power of two, so that fp16
// keeps 11 bits for every row; adding e_f to the exponent restores the product.
// Each role walks its tiles with a cursor that advances by additions (no division by a
// runtime value on the per-tile or per-block path).
//
// Both kernels are launched with programmatic dependent launch (launch.cuh): they let the
// next kernel on the stream be scheduled at once and wait (griddepcontrol.wait) only before
// storing the partial state (key pass) or loading the first state image (query pass).
//
// Every mbarrier wait is bounded (2 s); a CTA that gives up raises the device
// error word, stops issuing work, drains its own copies and frees its TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "favor_internal.h"
#include "launch.cuh"
#include "sm100_ptx.cuh"

namespace favor {

__device__ unsigned int g_sm100_error_word;

namespace {
using namespace sm100;

constexpr int kThreads = 384;  // key pass: producer, MMA, two norm warps, 8 epilogue warps
constexpr int kEpiWarp0 = 4;
constexpr int kEpiThreads = 256;
constexpr uint32_t kBarEpi = 1;    // named barrier: epilogue max exchange (lock-step key pass)
constexpr float kTau = 8.f;        // lazy stabiliser threshold (log2 units)
// registers per thread after setmaxnreg: producer / MMA warpgroup, epilogue warpgroups
constexpr int kRegsLow = 88, kRegsHigh = 200;

__device__ __forceinline__ uint32_t taddr(uint32_t base, int lane_quarter, int col) {
  return base + (static_cast<uint32_t>(lane_quarter * 32) << 16) + static_cast<uint32_t>(col);
}

// Multiplies `chunks` x 8 consecutive TMEM columns of this warp's 32 lanes by `sc` (per lane).
// A cold path (a raised stabiliser), kept out of line so it costs the hot loop no registers.
__device__ __noinline__ void scale_tmem_row(uint32_t taddr0, int chunks, float sc) {
  for (int cc = 0; cc < chunks; ++cc) {
    uint32_t v[8];
    tmem_ld8(taddr0 + 8 * cc, v);
    tmem_wait_ld();
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) * sc);
    tmem_st8(taddr0 + 8 * cc, v);
  }
  tmem_wait_st();
}

// ============================================================================
// Key pass, d = 128: lock-step (both epilogue warpgroups on every tile)
// ============================================================================
template <int D>
struct KeyCfg {
  static constexpr int NST = (D == 64) ? 4 : 2;   // K/V pipeline stages
  static constexpr int NB1 = (D == 64) ? 2 : 1;   // U^T buffers in TMEM
  static constexpr int RGN = 128 * 64 * 2;        // one 128-token x 64-dim swizzled region
  static constexpr int TILE = RGN * (D / 64);     // one K (or V) tile
  static constexpr int NS = D + 16;               // S columns: D values, then the ones block
  // TMEM columns
  static constexpr int T_WHI = 0;
  static constexpr int T_WLO = D / 2;
  static constexpr int T_D1 = D;
  static constexpr int T_S = D + NB1 * 128;
  static_assert(T_S + NS <= 512, "TMEM budget");
  // shared memory, from a 1024-aligned base
  static constexpr int S_K = 0;
  static constexpr int S_V = S_K + NST * TILE;
  static constexpr int S_ONES = S_V + NST * TILE;  // 2 atoms x 16 rows x 128 B
  static constexpr int S_NRM = S_ONES + 4096;      // NST x 128 floats
  static constexpr int S_RED = S_NRM + NST * 512;  // 2 x 8 floats
  static constexpr int S_BAR = S_RED + 64;
  // barriers: kv_full[NST], kv_empty[NST], nrm_ready[NST], d1_full[NB1], phi_ready[NB1], s_done
  static constexpr int B_KVF = 0, B_KVE = NST, B_NRM = 2 * NST, B_D1F = 3 * NST, B_PHI = 3 * NST + NB1,
                       B_SDONE = 3 * NST + 2 * NB1, NBAR = 3 * NST + 2 * NB1 + 1;
  static constexpr int S_TPTR = S_BAR + NBAR * 8;
  static constexpr int S_ABORT = S_TPTR + 8;
  static constexpr int SMEM = S_ABORT + 16 + 1024;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1) key_pass_sm100(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const float* __restrict__ W,
    float* __restrict__ part_S, float* __restrict__ part_c, int L, int m, int P, int chunk, int nsb, float wscale,
    float nscale) {
  using C = KeyCfg<D>;
  extern __shared__ unsigned char smem_raw[];
  griddep_launch_dependents();  // the next kernel on the stream may be scheduled as SMs free up
  // offset the __shared__ array itself (not via an integer cast), so that every pointer derived
  // from it stays a shared-memory pointer and compiles to shared loads and stores
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // the feature groups of one (kv head, chunk) are adjacent CTAs, so they run together and the
  // second group's K/V reads hit L2
  const int grp = blockIdx.x, p = blockIdx.y, head = blockIdx.z;
  const int f0 = grp * 128, gw = min(128, m - f0);
  const int t_begin = p * chunk, t_end = min(L, t_begin + chunk);
  const int ntiles = (t_end - t_begin + 127) / 128;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::S_ABORT);
  uint32_t* tptr_slot = reinterpret_cast<uint32_t*>(smem + C::S_TPTR);
  float* nrm = reinterpret_cast<float*>(smem + C::S_NRM);
  float* red = reinterpret_cast<float*>(smem + C::S_RED);
  auto bar = [&](int i) { return sbase + C::S_BAR + 8u * i; };

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(bar(C::B_KVF + s), 1);
      mbar_init(bar(C::B_KVE + s), 1);
      mbar_init(bar(C::B_NRM + s), 2);
    }
    for (int b = 0; b < C::NB1; ++b) {
      mbar_init(bar(C::B_D1F + b), 1);
      mbar_init(bar(C::B_PHI + b), kEpiThreads / 32);
    }
    mbar_init(bar(C::B_SDONE), 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tptr_slot), 512);
    tmem_relinquish();
  }
  // ones tile: K-major [16 rows x 128 tokens] in two 64-token atoms; row 0 = 1.0, rows 1..15 = 0
  for (int i = tid; i < 4096 / 4; i += kThreads) {
    const int row = (i * 4 % 2048) / 128;
    reinterpret_cast<uint32_t*>(smem + C::S_ONES)[i] = (row == 0) ? 0x3F803F80u : 0u;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tptr_slot;

  const bool epi = warp >= kEpiWarp0;
  const int eq = warp & 3;                   // TMEM lane quarter of this warp
  const int ewg = (warp - kEpiWarp0) >> 2;   // epilogue warpgroup: 0 or 1
  const int frow = eq * 32 + lane;           // feature row (TMEM lane) owned by an epilogue thread
  const bool fvalid = frow < gw;

  if (epi) {  // W' = hi + lo (bf16) into TMEM as the A operand of MMA1: lane = feature, 2 dims per column
    const int f = f0 + frow;
    uint32_t words[32];
#pragma unroll
    for (int half = 0; half < D / 64; ++half) {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float w0 = 0.f, w1 = 0.f;
        if (fvalid) {
          const float2 v = *reinterpret_cast<const float2*>(W + static_cast<size_t>(f) * D + half * 64 + 2 * j);
          w0 = v.x * wscale;
          w1 = v.y * wscale;
        }
        if (ewg == 0) {
          words[j] = pack_bf16x2(w0, w1);
        } else {
          const float h0 = __bfloat162float(__float2bfloat16_rn(w0));
          const float h1 = __bfloat162float(__float2bfloat16_rn(w1));
          words[j] = pack_bf16x2(w0 - h0, w1 - h1);
        }
      }
      tmem_st32(taddr(tbase, eq, (ewg == 0 ? C::T_WHI : C::T_WLO) + half * 32), words);
    }
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  unsigned int* err = &g_sm100_error_word;
  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % C::NST;
        if (i >= C::NST && !mbar_wait(bar(C::B_KVE + s), ((i / C::NST) - 1) & 1, abort_flag, err)) break;
        mbar_arrive_expect_tx(bar(C::B_KVF + s), 2 * C::TILE);
        const int t0 = t_begin + 128 * i;
#pragma unroll
        for (int r = 0; r < D / 64; ++r) {
          tma_load_3d(sbase + C::S_K + s * C::TILE + r * C::RGN, &tmK, bar(C::B_KVF + s), 64 * r, t0, head);
          tma_load_3d(sbase + C::S_V + s * C::TILE + r * C::RGN, &tmV, bar(C::B_KVF + s), 64 * r, t0, head);
        }
        issued = i + 1;
      }
      // drain: every load this CTA issued must have landed before it exits
      for (int i = max(0, issued - C::NST); i < issued; ++i)
        mbar_wait(bar(C::B_KVF + i % C::NST), (i / C::NST) & 1, abort_flag, err, 200000000ull);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t id1 = idesc_bf16(128, 128, false, false);
      const uint32_t idv = idesc_bf16(128, D, false, true);
      const uint32_t ido = idesc_bf16(128, 16, false, false);
      bool ok = true;
      auto mma2 = [&](int j) {
        const int s = j % C::NST, b = j % C::NB1;
        if (!mbar_wait(bar(C::B_PHI + b), (j / C::NB1) & 1, abort_flag, err)) return false;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t a = tbase + C::T_D1 + 128 * b + 8 * ks;
          const uint64_t bv = sdesc_sw128(sbase + C::S_V + s * C::TILE + 2048 * ks, C::RGN, 1024);
          const uint64_t bo = sdesc_sw128(sbase + C::S_ONES + (ks >> 2) * 2048 + 32 * (ks & 3), 16, 1024);
          const uint32_t acc = (j > 0 || ks > 0) ? 1u : 0u;
          mma_ts(tbase + C::T_S, a, bv, idv, acc);
          mma_ts(tbase + C::T_S + D, a, bo, ido, acc);
        }
        mma_commit(bar(C::B_KVE + s));
        mma_commit(bar(C::B_SDONE));
        return true;
      };
      for (int i = 0; i < ntiles && ok; ++i) {
        const int s = i % C::NST, b = i % C::NB1;
        if (!mbar_wait(bar(C::B_KVF + s), (i / C::NST) & 1, abort_flag, err)) break;
        if (i >= C::NB1 && !mbar_wait(bar(C::B_SDONE), (i - C::NB1) & 1, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t d1 = tbase + C::T_D1 + 128 * b;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t bk = sdesc_sw128(sbase + C::S_K + s * C::TILE + (ks >> 2) * C::RGN + 32 * (ks & 3), 16, 1024);
          mma_ts(d1, tbase + C::T_WHI + 8 * ks, bk, id1, ks > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t bk = sdesc_sw128(sbase + C::S_K + s * C::TILE + (ks >> 2) * C::RGN + 32 * (ks & 3), 16, 1024);
          mma_ts(d1, tbase + C::T_WLO + 8 * ks, bk, id1, 1u);
        }
        mma_commit(bar(C::B_D1F + b));
        if (C::NB1 == 2 && i >= 1) ok = mma2(i - 1);
        if (C::NB1 == 1) ok = mma2(i);
      }
      if (ok && C::NB1 == 2 && ntiles >= 1 && !*abort_flag) mma2(ntiles - 1);
      // all MMAs of this CTA complete before TMEM is released
      mbar_wait(bar(C::B_SDONE), (ntiles - 1) & 1, abort_flag, err, 200000000ull);
    }
  } else if (warp == 2 || warp == 3) {
    // ---------------- key norms: n(k) = |k|^2 * nscale, +inf past the chunk end ----------------
    // two warps, two tokens per lane each; the 16-byte chunks of a swizzled row are summed in
    // any order, and four accumulators keep the FMA chains short
    const int wsel = warp - 2;
    for (int i = 0; i < ntiles; ++i) {
      const int s = i % C::NST;
      if (!mbar_wait(bar(C::B_KVF + s), (i / C::NST) & 1, abort_flag, err)) break;
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        const int t = lane + 32 * (2 * qq + wsel);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int r = 0; r < D / 64; ++r) {
          const uint4* row = reinterpret_cast<const uint4*>(smem + C::S_K + s * C::TILE + r * C::RGN + t * 128);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 v = row[c ^ (t & 7)];  // lanes of a wavefront start on different banks
            const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float lo = __uint_as_float(wv[k] << 16), hi = __uint_as_float(wv[k] & 0xFFFF0000u);
              acc[k] = fmaf(lo, lo, acc[k]);
              acc[k] = fmaf(hi, hi, acc[k]);
            }
          }
        }
        const float sum = (acc[0] + acc[1]) + (acc[2] + acc[3]);
        nrm[s * 128 + t] = (t_begin + 128 * i + t < t_end) ? sum * nscale : INFINITY;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_NRM + s));
    }
  } else if (epi) {
    // ---------------- epilogue: exp feature map, stabiliser, state readout ----------------
    float c_run = -INFINITY;
    for (int i = 0; i < ntiles; ++i) {
      const int s = i % C::NST, b = i % C::NB1;
      mbar_wait(bar(C::B_D1F + b), (i / C::NB1) & 1, abort_flag, err);
      mbar_wait(bar(C::B_NRM + s), (i / C::NST) & 1, abort_flag, err);
      tc_fence_after();
      uint32_t u[64];
      {
        uint32_t r0[32], r1[32];
        tmem_ld32(taddr(tbase, eq, C::T_D1 + 128 * b + 64 * ewg), r0);
        tmem_ld32(taddr(tbase, eq, C::T_D1 + 128 * b + 64 * ewg + 32), r1);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          u[k] = r0[k];
          u[32 + k] = r1[k];
        }
      }
      const float4* nv = reinterpret_cast<const float4*>(nrm + s * 128 + 64 * ewg);
      float a[64];
      float mx = -INFINITY;
#pragma unroll
      for (int k4 = 0; k4 < 16; ++k4) {
        const float4 n4 = nv[k4];
        a[4 * k4 + 0] = __uint_as_float(u[4 * k4 + 0]) - n4.x;
        a[4 * k4 + 1] = __uint_as_float(u[4 * k4 + 1]) - n4.y;
        a[4 * k4 + 2] = __uint_as_float(u[4 * k4 + 2]) - n4.z;
        a[4 * k4 + 3] = __uint_as_float(u[4 * k4 + 3]) - n4.w;
      }
      if (fvalid) {
#pragma unroll
        for (int k = 0; k < 64; ++k) mx = fmaxf(mx, a[k]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (lane == 0) red[(i & 1) * 8 + (warp - kEpiWarp0)] = mx;
      named_bar_sync(kBarEpi, kEpiThreads);
      float M = red[(i & 1) * 8];
#pragma unroll
      for (int w = 1; w < 8; ++w) M = fmaxf(M, red[(i & 1) * 8 + w]);
      if (c_run == -INFINITY) {
        c_run = M;
      } else if (M > c_run + kTau) {  // uniform across the CTA: rescale S to the new stabiliser
        mbar_wait(bar(C::B_SDONE), (i - 1) & 1, abort_flag, err);
        tc_fence_after();
        const float sc = ex2(c_run - M);
#pragma unroll
        for (int cc = 0; cc < C::NS / 16; ++cc) {
          const int col = C::T_S + ewg * (C::NS / 2) + 8 * cc;
          uint32_t v[8];
          tmem_ld8(taddr(tbase, eq, col), v);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 8; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) * sc);
          tmem_st8(taddr(tbase, eq, col), v);
        }
        tmem_wait_st();
        c_run = M;
      }
      uint32_t wph[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float p0 = fvalid ? ex2(a[2 * j] - c_run) : 0.f;
        const float p1 = fvalid ? ex2(a[2 * j + 1] - c_run) : 0.f;
        wph[j] = pack_bf16x2(p0, p1);
      }
      tmem_st32(taddr(tbase, eq, C::T_D1 + 128 * b + 32 * ewg), wph);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_PHI + b));
    }
    // state readout: S rows of this group -> partial [m][D+1], once the kernels before this
    // one on the stream (which may read the partial state) have completed
    griddep_wait();
    mbar_wait(bar(C::B_SDONE), (ntiles - 1) & 1, abort_flag, err);
    tc_fence_after();
    float* outp = part_S + (static_cast<size_t>(head) * P + p) * static_cast<size_t>(m) * (D + 1);
#pragma unroll
    for (int cc = 0; cc < C::NS / 16; ++cc) {
      const int col0 = ewg * (C::NS / 2) + 8 * cc;
      uint32_t v[8];
      tmem_ld8(taddr(tbase, eq, C::T_S + col0), v);
      tmem_wait_ld();
      if (fvalid) {
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (col0 + k <= D) outp[static_cast<size_t>(f0 + frow) * (D + 1) + col0 + k] = __uint_as_float(v[k]);
      }
    }
    if (ewg == 0 && fvalid) part_c[(static_cast<size_t>(head) * P + p) * nsb + f0 + frow] = c_run;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, 512);
}

// ============================================================================
// Key pass, d = 64: two epilogue warpgroups, each with its own projection, weights and accumulator
// ============================================================================
// Each warpgroup owns a U^T buffer, a phi buffer and an S accumulator in tensor
// memory, its own running stabilisers and its own MMA-issuing thread (warp 1 for
// warpgroup 0, warp 2 for warpgroup 1).  The epilogue releases U^T as soon as it
// has read it, so the next tile's projection runs while this tile's exponentials
// and its contraction finish; phi goes to its own buffer.  Warp 3 computes every
// tile's key norms as soon as the tile lands, once for both warpgroups.  The
// normaliser column sum_t phi is accumulated by the epilogue itself, in fp32.
//  * WIDE (m > 128): a CTA covers 256 features; warpgroup w takes features 128 w ..
//    128 w + 127 of every tile, so each K/V tile and its norms serve 256 features and
//    the grid is half as large.
//  * otherwise: a CTA covers 128 features; the warpgroups take alternate tiles, and at
//    the end the two accumulators are merged exactly: S = 2^(c0-c) S0 + 2^(c1-c) S1.
template <bool WIDE>
struct KeyPP {
  static constexpr int D = 64;
  static constexpr int NFEAT = WIDE ? 256 : 128;  // features per CTA
  // warp 0 TMA producer, warps 1-2 MMA issuers, warp 3 key norms, warps 4-11 two epilogue
  // warpgroups (each covers the four TMEM lane quarters once, as warp % 4)
  static constexpr int THREADS = 384;
  static constexpr int EPI0 = 4;
  static constexpr int NST = WIDE ? 4 : 5;  // K/V stages (the wide W' takes the fifth's room)
  static constexpr int TILE = 128 * 64 * 2;
  // TMEM columns: warpgroup w owns U^T at 256 w, phi at 256 w + 128 (bf16 pairs), S at 256 w + 192
  static constexpr int T_U = 0, T_P = 128, T_S = 192, T_STRIDE = 256;
  // W' = hi + lo in bf16, each NFEAT features x 64 dims, K-major SW128 (the A operands of MMA1;
  // warpgroup w of a wide CTA starts at row 128 w)
  static constexpr int S_WHI = 0, S_WLO = NFEAT * 128;
  static constexpr int S_K = S_WLO + NFEAT * 128;
  static constexpr int S_V = S_K + NST * TILE;
  // per stage: n(k) of the tile's 128 tokens as bf16 hi, mid, lo (then 13 zeros), K-major with the
  // 32-byte swizzle: the B operand of one more projection step against S_NA, whose rows are
  // (-1, -1, -1, 0, ...), so that U^T comes out of the tensor core as W'k - n(k)
  static constexpr int S_NB = S_V + NST * TILE;
  static constexpr int S_NA = S_NB + NST * 4096;
  static constexpr int S_CW = S_NA + 4096;          // final stabilisers and normalisers, [2][2][128]
  static constexpr int S_BAR = S_CW + 2048;
  // PHI and SDONE come in halves per warpgroup (2 w + h): the weights of tokens 64 h .. 64 h + 63
  // and the contraction steps that read them
  static constexpr int B_KVF = 0, B_KVE = NST, B_NRM = 2 * NST, B_D1F = B_NRM + NST, B_UE = B_D1F + 2,
                       B_PHI = B_UE + 2, B_SDONE = B_PHI + 4, NBAR = B_SDONE + 4;
  static constexpr int S_TPTR = S_BAR + NBAR * 8;
  static constexpr int S_ABORT = S_TPTR + 8;
  static constexpr int SMEM = S_ABORT + 16 + 1024;
  static_assert(SMEM <= 232448, "shared memory budget");
};

// RELU: the feature map max(W'k, 0) instead of 2^(W'k - n(k) - c) (W' then carries no log2(e)): no
// norms, no stabilisers (written as 0, so the reduction sums the chunks as they are), no rescale.
template <bool WIDE, bool RELU>
__global__ void __launch_bounds__(KeyPP<WIDE>::THREADS, 1) key_pass_pp_sm100(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const float* __restrict__ W,
    float* __restrict__ part_S, float* __restrict__ part_c, int L, int m, int P, int chunk, int nsb, float wscale,
    float nscale) {
  using C = KeyPP<WIDE>;
  constexpr int D = C::D;
  extern __shared__ unsigned char smem_raw[];
  griddep_launch_dependents();  // the next kernel on the stream may be scheduled as SMs free up
  // offset the __shared__ array itself (not via an integer cast), so that every pointer derived
  // from it stays a shared-memory pointer and compiles to shared loads and stores
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = blockIdx.x, p = blockIdx.y, head = blockIdx.z;
  const int f0 = grp * C::NFEAT, gw = min(C::NFEAT, m - f0);
  const int t_begin = p * chunk, t_end = min(L, t_begin + chunk);
  const int ntiles = (t_end - t_begin + 127) / 128;
  // tiles of warpgroup w: all of them (wide), or w, w + 2, ...
  constexpr int TSTEP = WIDE ? 1 : 2;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::S_ABORT);
  uint32_t* tptr_slot = reinterpret_cast<uint32_t*>(smem + C::S_TPTR);
  float* cw = reinterpret_cast<float*>(smem + C::S_CW);
  auto bar = [&](int i) { return sbase + C::S_BAR + 8u * i; };

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(bar(C::B_KVF + s), 1);
      mbar_init(bar(C::B_KVE + s), WIDE ? 2 : 1);  // the contraction(s) of the stage's tile
      mbar_init(bar(C::B_NRM + s), 1);  // the norm warp, once per tile of the stage
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(bar(C::B_D1F + w), 1);
      mbar_init(bar(C::B_UE + w), 4);
      for (int h = 0; h < 2; ++h) {
        mbar_init(bar(C::B_PHI + 2 * w + h), 4);
        mbar_init(bar(C::B_SDONE + 2 * w + h), 1);
      }
    }
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    // the first stages' loads go out now, under the W' fill below
    for (int i = 0; i < min(ntiles, C::NST); ++i) {
      mbar_arrive_expect_tx(bar(C::B_KVF + i), 2 * C::TILE);
      tma_load_3d(sbase + C::S_K + i * C::TILE, &tmK, bar(C::B_KVF + i), 0, t_begin + 128 * i, head);
      tma_load_3d(sbase + C::S_V + i * C::TILE, &tmV, bar(C::B_KVF + i), 0, t_begin + 128 * i, head);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tptr_slot), 512);
    tmem_relinquish();
  }
  // W' = hi + lo (bf16) as the K-major 128B-swizzled A operands of MMA1: row f, 16-byte chunk c
  // at c ^ (f % 8); the pair keeps ~16 bits of W', so the exponents stay within the bf16
  // output tolerance on heavy-tailed keys
  for (int item = tid; item < C::NFEAT * 8; item += C::THREADS) {
    const int f = item >> 3, c = item & 7;
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float w0 = 0.f, w1 = 0.f;
      if (f < gw) {
        const float2 v = *reinterpret_cast<const float2*>(W + static_cast<size_t>(f0 + f) * D + 8 * c + 2 * k);
        w0 = v.x * wscale;
        w1 = v.y * wscale;
      }
      hi[k] = pack_bf16x2(w0, w1);
      lo[k] = pack_bf16x2(w0 - __uint_as_float(hi[k] << 16), w1 - __uint_as_float(hi[k] & 0xFFFF0000u));
    }
    const int off = f * 128 + ((c ^ (f & 7)) << 4);
    *reinterpret_cast<uint4*>(smem + C::S_WHI + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(smem + C::S_WLO + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
  // the norm step's A operand (row r, 16-byte chunk c at c ^ (r / 4 % 2)) and its B operands' zero
  // chunks (the norm warp writes chunk 0 of each row per tile)
  for (int r = tid; r < 128; r += C::THREADS) {
    const int sw = (r >> 2) & 1;
    *reinterpret_cast<uint4*>(smem + C::S_NA + r * 32 + (sw << 4)) = make_uint4(0xBF80BF80u, 0x0000BF80u, 0u, 0u);
    *reinterpret_cast<uint4*>(smem + C::S_NA + r * 32 + ((1 ^ sw) << 4)) = make_uint4(0u, 0u, 0u, 0u);
  }
  for (int i = tid; i < C::NST * 128; i += C::THREADS) {
    const int r = i & 127;
    *reinterpret_cast<uint4*>(smem + C::S_NB + (i >> 7) * 4096 + r * 32 + ((1 ^ ((r >> 2) & 1)) << 4)) = make_uint4(0u, 0u, 0u, 0u);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tptr_slot;
  unsigned int* err = &g_sm100_error_word;

  // registers: the producer / MMA warpgroup gives part of its share to the two epilogue
  // warpgroups (128 x 88 + 256 x 200 = 62464 <= 384 x 168, the launch allocation; the host
  // checks the compiled count before launching)
  if (warp < C::EPI0) {
  setmaxnreg_dec<kRegsLow>();
  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int issued = min(ntiles, C::NST);  // issued during the set-up
      for (int i = issued; i < ntiles; ++i) {
        const int s = i % C::NST;
        if (!mbar_wait<true>(bar(C::B_KVE + s), ((i / C::NST) - 1) & 1, abort_flag, err)) break;
        mbar_arrive_expect_tx(bar(C::B_KVF + s), 2 * C::TILE);
        const int t0 = t_begin + 128 * i;
        tma_load_3d(sbase + C::S_K + s * C::TILE, &tmK, bar(C::B_KVF + s), 0, t0, head);
        tma_load_3d(sbase + C::S_V + s * C::TILE, &tmV, bar(C::B_KVF + s), 0, t0, head);
        issued = i + 1;
      }
      for (int i = max(0, issued - C::NST); i < issued; ++i)
        mbar_wait(bar(C::B_KVF + i % C::NST), (i / C::NST) & 1, abort_flag, err, 200000000ull);
    }
  } else if (warp == 1 || warp == 2) {
    // ---------------- MMA issuer of warpgroup w: its tiles (all, or w, w + 2, ...) ----------------
    // The next tile's projection is issued as soon as the epilogue has read this tile's
    // U^T, ahead of this tile's contraction.
    if (lane == 0) {
      const int w = warp - 1;
      const uint32_t id1 = idesc_bf16(128, 128, false, false);
      const uint32_t idv = idesc_bf16(128, D, false, true);  // V tile as an MN-major B operand
      const uint32_t dU = tbase + w * C::T_STRIDE + C::T_U, dP = tbase + w * C::T_STRIDE + C::T_P,
                     dS = tbase + w * C::T_STRIDE + C::T_S;
      const uint32_t wrow = WIDE ? w * 128 * 128 : 0;  // this warpgroup's rows of W'
      auto mma1 = [&](int i) {  // U^T = (W'hi + W'lo) K^T (- n(k), once the tile's norms are in)
        const int s = i % C::NST;
#pragma unroll
        for (int ks = 0; ks < 2 * (D / 16); ++ks) {
          const int kk = ks % (D / 16);
          mma_ss(dU, sdesc_sw128(sbase + (ks < D / 16 ? C::S_WHI : C::S_WLO) + wrow + 32 * kk, 16, 1024),
                 sdesc_sw128(sbase + C::S_K + s * C::TILE + 32 * kk, 16, 1024), id1, ks > 0 ? 1u : 0u);
        }
        if constexpr (!RELU) {
          if (!mbar_wait(bar(C::B_NRM + s), (i / C::NST) & 1, abort_flag, err)) return false;
          tc_fence_after();
          mma_ss(dU, sdesc_sw32(sbase + C::S_NA, 256), sdesc_sw32(sbase + C::S_NB + s * 4096, 256), id1, 1u);
        }
        mma_commit(bar(C::B_D1F + w));
        return true;
      };
      int cnt = 0;
      const int first = WIDE ? 0 : w;
      bool ok = first < ntiles && mbar_wait(bar(C::B_KVF + first % C::NST), (first / C::NST) & 1, abort_flag, err);
      if (ok) {
        tc_fence_after();
        ok = mma1(first);
      }
      for (int i = first; i < ntiles && ok; i += TSTEP, ++cnt) {
        const int s = i % C::NST;
        if (i + TSTEP < ntiles) {
          if (!mbar_wait(bar(C::B_UE + w), cnt & 1, abort_flag, err)) break;  // U^T of tile i read
          const int s2 = (i + TSTEP) % C::NST;
          if (!mbar_wait(bar(C::B_KVF + s2), ((i + TSTEP) / C::NST) & 1, abort_flag, err)) break;  // the next tile landed
          tc_fence_after();
          if (!mma1(i + TSTEP)) break;
        }
        // MMA2: S_w += phi^T V, 16 tokens per step, each half of the tile as soon as its weights are in
        for (int h = 0; h < 2 && ok; ++h) {
          if (!(ok = mbar_wait(bar(C::B_PHI + 2 * w + h), cnt & 1, abort_flag, err))) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int ks = 4 * h + k;
            const uint64_t bv = sdesc_sw128(sbase + C::S_V + s * C::TILE + 2048 * ks, 16, 1024);
            mma_ts(dS, dP + 8 * ks, bv, idv, (cnt > 0 || ks > 0) ? 1u : 0u);
          }
          if (h == 1) mma_commit(bar(C::B_KVE + s));
          mma_commit(bar(C::B_SDONE + 2 * w + h));
        }
      }
      const int mine = WIDE ? ntiles : (ntiles + 1 - w) / 2;
      if (mine > 0) mbar_wait(bar(C::B_SDONE + 2 * w + 1), (mine - 1) & 1, abort_flag, err, 200000000ull);
    }
  } else {
    // ---------------- key norms: n(k) = |k|^2 nscale per token (2^100 past the chunk end) ----------------
    // Lane l takes tokens l, l + 32, l + 64, l + 96 of each tile, two at a time.  The 16-byte chunks of a swizzled
    // row are summed in any order; token t starts at chunk t % 8, so the eight lanes of a
    // shared-memory wavefront hit different banks.  The norms go to the stage's operand of the
    // projection's norm step (S_NB), read by the tensor cores once the issuer has seen them
    // published.  The stage's norms are overwritten only after the tile that last used it has
    // been contracted, which comes after its projection (one thread's MMAs run in issue order),
    // so no other wait is needed.
    for (int i = 0; i < (RELU ? 0 : ntiles); ++i) {
      const int s = i % C::NST;
      if (!mbar_wait(bar(C::B_KVF + s), (i / C::NST) & 1, abort_flag, err)) break;
#pragma unroll 1
      for (int r2 = 0; r2 < 2; ++r2) {  // two tokens at a time, for independent chains
        const int ta = lane + 64 * r2, tb = ta + 32;
        const uint4* ra = reinterpret_cast<const uint4*>(smem + C::S_K + s * C::TILE + ta * 128);
        const uint4* rb = reinterpret_cast<const uint4*>(smem + C::S_K + s * C::TILE + tb * 128);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 va = ra[c ^ (ta & 7)], vb = rb[c ^ (tb & 7)];
          const uint32_t wa[4] = {va.x, va.y, va.z, va.w}, wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 xa = make_float2(__uint_as_float(wa[q] << 16), __uint_as_float(wa[q] & 0xFFFF0000u));
            const float2 xb = make_float2(__uint_as_float(wb[q] << 16), __uint_as_float(wb[q] & 0xFFFF0000u));
            acc[q & 1] = __ffma2_rn(xa, xa, acc[q & 1]);
            acc[2 + (q & 1)] = __ffma2_rn(xb, xb, acc[2 + (q & 1)]);
          }
        }
        const float sa = (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y);
        const float sb = (acc[2].x + acc[2].y) + (acc[3].x + acc[3].y);
        // n(k) as bf16 hi + mid + lo (exact residuals, ~24 bits); a token past the chunk end gets
        // n = 2^100, which sends its exponent to -2^100 and its weight to 0
        auto put = [&](int t, float nk) {
          const uint32_t h = pack_bf16x2(nk, 0.f);
          const float r1 = nk - __uint_as_float(h << 16);
          const uint32_t hm = pack_bf16x2(nk, r1);
          const float r2 = r1 - __uint_as_float(hm & 0xFFFF0000u);
          *reinterpret_cast<uint4*>(smem + C::S_NB + s * 4096 + t * 32 + (((t >> 2) & 1) << 4)) =
              make_uint4(hm, pack_bf16x2(r2, 0.f), 0u, 0u);
        };
        put(ta, (t_begin + 128 * i + ta < t_end) ? sa * nscale : 0x1p100f);
        put(tb, (t_begin + 128 * i + tb < t_end) ? sb * nscale : 0x1p100f);
      }
      fence_proxy_async_smem();  // the norms are read by the tensor cores
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_NRM + s));  // release: the 128 norms are stored
    }
  }
  } else {
    setmaxnreg_inc<kRegsHigh>();
    // ---------------- epilogue warpgroup ewg: its tiles (all, or ewg, ewg + 2, ...) ----------------
    const int eq = warp & 3;
    const int ewg = (warp - C::EPI0) >> 2;
    const int frow = eq * 32 + lane;                  // the thread's TMEM lane (row of U^T and S)
    const int fr = (WIDE ? 128 * ewg : 0) + frow;     // its feature, counted from f0
    const bool fvalid = fr < gw;
    // Each thread owns feature f0 + fr and reads each U^T value of its row once.  Its
    // stabiliser c is that feature's running max exponent over the tiles seen so far,
    // raised (with an exact rescale of its S row and normaliser) only when a tile exceeds
    // it by more than 2^kTau, and never below floor = |w|^2 log2(e)/2 - 64: by completing
    // the square no exponent of this feature exceeds |w|^2 log2(e)/2, so no phi exceeds
    // 2^64 and the fp32 state cannot overflow for any |v| < 2^46 at any sequence length up
    // to 2^17.
    float floor_c;
    {
      float w2 = 0.f;
      if (fvalid) {
        const float4* wr = reinterpret_cast<const float4*>(W + static_cast<size_t>(f0 + fr) * D);
#pragma unroll
        for (int k = 0; k < D / 4; ++k) {
          const float4 v = wr[k];
          w2 = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, w2))));
        }
      }
      floor_c = RELU ? 0.f : w2 * static_cast<float>(kLog2e * 0.5) - 64.f;
    }
    float c_run = floor_c, tmax = -INFINITY, zsum = 0.f;  // zsum: this feature's normaliser sum_t phi
    const uint32_t cU = ewg * C::T_STRIDE + C::T_U, cP = ewg * C::T_STRIDE + C::T_P,
                   cS = ewg * C::T_STRIDE + C::T_S;
    int cnt = 0;
    for (int i = WIDE ? 0 : ewg; i < ntiles; i += TSTEP, ++cnt) {
      const int s = i % C::NST;
      mbar_wait(bar(C::B_D1F + ewg), cnt & 1, abort_flag, err);
      // the norms of tile i (the norm warp cannot have moved on to the stage's next tile: that
      // tile is loaded only after this one has been contracted)
      // this tile's U^T row into registers (one read), then release it to the next projection
      float ut[128];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) tmem_ld32(taddr(tbase, eq, cU + 32 * q4), *reinterpret_cast<uint32_t(*)[32]>(&ut[32 * q4]));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_UE + ewg));
      // the previous tile raised the running max: rescale S and the normaliser now, once the
      // previous tile's contraction is complete
      const bool need = !RELU && tmax > c_run + kTau;
      if (__any_sync(0xffffffffu, need)) {
        if (cnt >= 1) mbar_wait(bar(C::B_SDONE + 2 * ewg + 1), (cnt - 1) & 1, abort_flag, err);
        tc_fence_after();
        scale_tmem_row(taddr(tbase, eq, cS), D / 8, need ? ex2(c_run - tmax) : 1.f);
      }
      if (need) {
        zsum *= ex2(c_run - tmax);
        c_run = tmax;
      }
      const float2 ncc = make_float2(-c_run, -c_run);
      float2 zs2 = make_float2(0.f, 0.f);
      float tm4[4] = {tmax, -INFINITY, -INFINITY, -INFINITY};  // four independent max chains
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        if ((q4 & 1) == 0) {  // a new half: its phi columns are free once the previous tile's
          const int h = q4 >> 1;  // contraction steps that read them are complete
          if (cnt >= 1) mbar_wait(bar(C::B_SDONE + 2 * ewg + h), (cnt - 1) & 1, abort_flag, err);
          tc_fence_after();
        }
        uint32_t wph[16];
#pragma unroll
        for (int k4 = 0; k4 < 8; ++k4) {  // two tokens per packed fp32x2 operation
          const float* r = &ut[32 * q4 + 4 * k4];
          float2 p01, p23;
          if constexpr (RELU) {
            p01 = make_float2(fmaxf(r[0], 0.f), fmaxf(r[1], 0.f));
            p23 = make_float2(fmaxf(r[2], 0.f), fmaxf(r[3], 0.f));
          } else {
            const float2 a01 = make_float2(r[0], r[1]), a23 = make_float2(r[2], r[3]);  // W'k - n(k)
            tm4[k4 & 3] = max3(tm4[k4 & 3], a01.x, a01.y);
            tm4[k4 & 3] = max3(tm4[k4 & 3], a23.x, a23.y);
            const float2 b01 = __fadd2_rn(a01, ncc), b23 = __fadd2_rn(a23, ncc);
            p01 = make_float2(ex2(b01.x), ex2(b01.y));
            p23 = make_float2(ex2(b23.x), ex2(b23.y));
          }
          zs2 = __fadd2_rn(zs2, __fadd2_rn(p01, p23));
          wph[2 * k4] = pack_bf16x2(p01.x, p01.y);
          wph[2 * k4 + 1] = pack_bf16x2(p23.x, p23.y);
        }
        // (a feature past m has W' = 0; its S row is computed but never written out)
        tmem_st16(taddr(tbase, eq, cP + 16 * q4), wph);  // phi, bf16 pairs
        if (q4 & 1) {  // this half's weights are in: its contraction steps may go
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(C::B_PHI + 2 * ewg + (q4 >> 1)));
        }
      }
      zsum += zs2.x + zs2.y;
      tmax = fmaxf(fmaxf(tm4[0], tm4[1]), fmaxf(tm4[2], tm4[3]));
    }
    if (!fvalid) zsum = 0.f;
    // write this group's partial state (merging the two accumulators row by row when they took
    // alternate tiles), once the kernels before this one on the stream (which may read the
    // partial state) have completed.  The rows go through shared memory (the K/V stages are free
    // once every MMA has completed) so that the partial state is written with coalesced 16-byte
    // stores; a row stride of D + 1 floats (odd) keeps the 32 rows of a warp on different banks.
    griddep_wait();
    float* stg = reinterpret_cast<float*>(smem + C::S_K);
    if constexpr (WIDE) {
      if (ntiles > 0) mbar_wait(bar(C::B_SDONE + 2 * ewg + 1), (ntiles - 1) & 1, abort_flag, err);
      tc_fence_after();
      named_bar_sync(3, 256);  // both warpgroups' contractions are complete: the stages may be reused
#pragma unroll
      for (int cc = 0; cc < D / 8; ++cc) {
        uint32_t v0[8];
        tmem_ld8(taddr(tbase, eq, ewg * C::T_STRIDE + C::T_S + 8 * cc), v0);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 8; ++k) stg[fr * (D + 1) + 8 * cc + k] = __uint_as_float(v0[k]);
      }
      stg[fr * (D + 1) + D] = zsum;
      if (fvalid) part_c[(static_cast<size_t>(head) * P + p) * nsb + f0 + fr] = c_run;
    } else {
    cw[ewg * 128 + frow] = c_run;
    cw[256 + ewg * 128 + frow] = zsum;
    named_bar_sync(3, 256);
    const int n0 = (ntiles + 1) / 2, n1 = ntiles / 2;  // tiles of each warpgroup
    const float c0 = cw[frow], c1 = cw[128 + frow];
    const float cmax = n1 > 0 ? fmaxf(c0, c1) : c0;
    if (n0 > 0) mbar_wait(bar(C::B_SDONE + 1), (n0 - 1) & 1, abort_flag, err);
    if (n1 > 0) mbar_wait(bar(C::B_SDONE + 3), (n1 - 1) & 1, abort_flag, err);
    tc_fence_after();
    const float s0 = n0 > 0 ? ex2(c0 - cmax) : 0.f, s1 = n1 > 0 ? ex2(c1 - cmax) : 0.f;
#pragma unroll
    for (int cc = 0; cc < D / 16; ++cc) {  // this warpgroup's half of the columns
      const int col0 = ewg * (D / 2) + 8 * cc;
      uint32_t v0[8], v1[8];
      tmem_ld8(taddr(tbase, eq, C::T_S + col0), v0);
      tmem_ld8(taddr(tbase, eq, C::T_STRIDE + C::T_S + col0), v1);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 8; ++k)
        stg[frow * (D + 1) + col0 + k] = fmaf(__uint_as_float(v1[k]), s1, __uint_as_float(v0[k]) * s0);
    }
    if (ewg == 0) {
      stg[frow * (D + 1) + D] = fmaf(cw[384 + frow], s1, cw[256 + frow] * s0);
      if (fvalid) part_c[(static_cast<size_t>(head) * P + p) * nsb + f0 + frow] = cmax;
    }
    }
    named_bar_sync(3, 256);
    // this group's rows f0 .. f0 + gw - 1 are contiguous in the partial state; gw (D + 1) is a
    // multiple of 16 floats since m and f0 are multiples of 16
    float4* outp = reinterpret_cast<float4*>(part_S + ((static_cast<size_t>(head) * P + p) * m + f0) * (D + 1));
    const float4* src = reinterpret_cast<const float4*>(stg);
    for (int i = tid - C::EPI0 * 32; i < gw * (D + 1) / 4; i += 256) outp[i] = src[i];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, 512);
}

// ============================================================================
// Linformer projections on the tensor cores (d = 64, bf16 K and V)
// ============================================================================
// Linformer notes page, "4 Model": E K and F V (k x d per kv head).  E and F (fp32) are first
// split into bf16 hi + lo (hi = bf16(x), lo = bf16(x - hi): about 16 bits of x).  One CTA takes
// (128 projected rows, key chunk, product, group of HPC kv heads): E is shared by the kv heads, so
// the K tiles of the group's heads sit side by side as one MN-major B operand (N = 64 HPC, one
// 64-column group per head) and each E tile serves them all.  It accumulates (Ehi + Elo)[rows,
// chunk] [K_h ...][chunk, :] in tensor memory (M = 128, 16 tokens per MMA), then writes the key
// pass's partial-state layout: F V with the constant column 1 on chunk 0 only (the reduction's sum
// is then 1) as head h, d^-1/4 E K as head heads + h, every stabiliser 0.
struct LinProj {
  static constexpr int D = 64;
  static constexpr int HPC = 4;  // kv heads per CTA
  // warp 0 TMA producer, warp 1 MMA issuer, warps 2-5 epilogue (TMEM lane quarter = warp % 4)
  static constexpr int THREADS = 192;
  static constexpr int NST = 3;                  // stages of TT tokens
  static constexpr int TT = 64;
  static constexpr int A_TILE = 128 * TT * 2;    // 128 rows x 64 tokens, bf16, K-major SW128
  static constexpr int B_TILE = TT * D * 2;      // one head: 64 tokens x 64 dims, bf16, MN-major SW128
  static constexpr int STAGE = 2 * A_TILE + HPC * B_TILE;  // E hi, E lo, the heads' K (or F, V)
  static constexpr int S_BAR = NST * STAGE;
  static constexpr int B_FULL = 0, B_EMPTY = NST, B_DONE = 2 * NST, NBAR = 2 * NST + 1;
  static constexpr int S_TPTR = S_BAR + NBAR * 8;
  static constexpr int S_ABORT = S_TPTR + 8;
  static constexpr int SMEM = S_ABORT + 16 + 1024;
  static constexpr int TCOLS = HPC * D;          // accumulator columns: 64 per head
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(A_TILE % 1024 == 0 && B_TILE % 1024 == 0, "swizzled operands on 1024-byte boundaries");
};

// [4][kpad][Lpad] bf16: E hi, E lo, F hi, F lo; rows kp .. kpad - 1 and tokens L .. Lpad - 1 are zero
// (Lpad, a multiple of 64, gives the rows the 16-byte stride a tensor map needs)
__global__ void split_hi_lo_kernel(const float* __restrict__ E, const float* __restrict__ F,
                                   __nv_bfloat16* __restrict__ out, int kp, int kpad, int L, int Lpad) {
  const size_t n = static_cast<size_t>(kpad) * Lpad;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int j = static_cast<int>(i / Lpad), t = static_cast<int>(i - static_cast<size_t>(j) * Lpad);
    const bool valid = j < kp && t < L;
    const size_t src = static_cast<size_t>(j) * L + t;
    const float e = valid ? E[src] : 0.f, f = valid ? F[src] : 0.f;
    const __nv_bfloat16 eh = __float2bfloat16_rn(e), fh = __float2bfloat16_rn(f);
    out[i] = eh;
    out[n + i] = __float2bfloat16_rn(e - __bfloat162float(eh));
    out[2 * n + i] = fh;
    out[3 * n + i] = __float2bfloat16_rn(f - __bfloat162float(fh));
  }
}

__global__ void __launch_bounds__(LinProj::THREADS, 1) linformer_proj_sm100(
    const __grid_constant__ CUtensorMap tmEF, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, float* __restrict__ part_S, float* __restrict__ part_c, int L, int kp,
    int P, int chunk, int nsb, int heads, float kscale) {
  using C = LinProj;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int mt = blockIdx.x, p = blockIdx.y;
  const int ngroups = (heads + C::HPC - 1) / C::HPC;
  const bool isE = static_cast<int>(blockIdx.z) >= ngroups;  // E K or F V of a group of kv heads
  const int h0 = (isE ? static_cast<int>(blockIdx.z) - ngroups : static_cast<int>(blockIdx.z)) * C::HPC;
  const int nh = min(C::HPC, heads - h0);  // the group's kv heads (the last group may be short)
  const int t_begin = p * chunk, t_end = min(L, t_begin + chunk);
  const int ntiles = (t_end - t_begin + C::TT - 1) / C::TT;  // chunk is a multiple of TT: only L cuts a stage
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::S_ABORT);
  uint32_t* tptr_slot = reinterpret_cast<uint32_t*>(smem + C::S_TPTR);
  auto bar = [&](int i) { return sbase + C::S_BAR + 8u * i; };
  unsigned int* err = &g_sm100_error_word;
  const int zs = isE ? 0 : 2;  // E hi, E lo at split index 0, 1; F at 2, 3
  const CUtensorMap* tmB = isE ? &tmK : &tmV;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(bar(C::B_FULL + s), 1);
      mbar_init(bar(C::B_EMPTY + s), 1);
    }
    mbar_init(bar(C::B_DONE), 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmEF);
    prefetch_tmap(tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tptr_slot), C::TCOLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tptr_slot;
  griddep_wait();  // the split of E and F is the kernel before this one

  if (warp == 0) {
    if (lane == 0) {  // ---------------- TMA producer ----------------
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % C::NST;
        if (i >= C::NST && !mbar_wait<true>(bar(C::B_EMPTY + s), ((i / C::NST) - 1) & 1, abort_flag, err)) break;
        const int t0 = t_begin + C::TT * i;
        const uint32_t st = sbase + s * C::STAGE;
        // the columns of absent heads (a short last group) are left as they are: computed, never written
        mbar_arrive_expect_tx(bar(C::B_FULL + s), 2 * C::A_TILE + nh * C::B_TILE);
        tma_load_3d(st, &tmEF, bar(C::B_FULL + s), t0, 128 * mt, zs);  // x = token, y = row, z = split
        tma_load_3d(st + C::A_TILE, &tmEF, bar(C::B_FULL + s), t0, 128 * mt, zs + 1);
        for (int n = 0; n < nh; ++n)  // x = dim, y = token, z = kv head
          tma_load_3d(st + 2 * C::A_TILE + n * C::B_TILE, tmB, bar(C::B_FULL + s), 0, t0, h0 + n);
        issued = i + 1;
      }
      for (int i = max(0, issued - C::NST); i < issued; ++i)  // no copy is in flight when the CTA leaves
        mbar_wait(bar(C::B_FULL + i % C::NST), (i / C::NST) & 1, abort_flag, err, 200000000ull);
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---------------- MMA issuer ----------------
      const uint32_t idesc = idesc_bf16(128, C::TCOLS, false, true);
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % C::NST;
        if (!mbar_wait(bar(C::B_FULL + s), (i / C::NST) & 1, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t st = sbase + s * C::STAGE;
#pragma unroll
        for (int kk = 0; kk < C::TT / 16; ++kk) {  // 16 tokens per step: Ehi then Elo against the same K rows
          // B: the heads' 64-column groups B_TILE bytes apart (LBO), 8-token groups 1024 apart (SBO)
          const uint64_t bd = sdesc_sw128(st + 2 * C::A_TILE + 2048 * kk, C::B_TILE, 1024);
          mma_ss(tbase, sdesc_sw128(st + 32 * kk, 16, 1024), bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
          mma_ss(tbase, sdesc_sw128(st + C::A_TILE + 32 * kk, 16, 1024), bd, idesc, 1u);
        }
        mma_commit(bar(C::B_EMPTY + s));
      }
      mma_commit(bar(C::B_DONE));  // arrives once every MMA above has completed
    }
  } else {  // ---------------- epilogue: one projected row per thread, for each head of the group ----------------
    const int eq = warp & 3;
    const int r = eq * 32 + lane, j = 128 * mt + r;
    const bool ok = mbar_wait(bar(C::B_DONE), 0, abort_flag, err, 200000000ull);
    tc_fence_after();
    const float sc = isE ? kscale : 1.f;
    const bool any = ok && ntiles > 0;  // no MMA wrote the accumulator otherwise
    for (int n = 0; n < nh; ++n) {
      uint32_t acc[64];
      tmem_ld32(taddr(tbase, eq, 64 * n), *reinterpret_cast<uint32_t(*)[32]>(&acc[0]));
      tmem_ld32(taddr(tbase, eq, 64 * n + 32), *reinterpret_cast<uint32_t(*)[32]>(&acc[32]));
      tmem_wait_ld();
      if (j < kp) {
        const int z = (isE ? heads : 0) + h0 + n;  // F V as head h, E K as head heads + h
        float* out = part_S + (static_cast<size_t>(z) * P + p) * static_cast<size_t>(kp) * (C::D + 1) +
                     static_cast<size_t>(j) * (C::D + 1);
#pragma unroll
        for (int c = 0; c < C::D; ++c) out[c] = any ? __uint_as_float(acc[c]) * sc : 0.f;
        out[C::D] = !isE && p == 0 ? 1.f : 0.f;
        part_c[(static_cast<size_t>(z) * P + p) * nsb + j] = 0.f;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, C::TCOLS);
}

// ============================================================================
// Query pass
// ============================================================================
// Where a query tile lies: query head bh (= b * H + h), 128-row tile qt within it, gq = bh % G and
// its state image, kv head bh / G (H = Hkv * G) counted from the CTA's first kv head.  Each role
// walks its tiles in fixed steps, so the cursor advances by additions: a division by a runtime
// value costs tens of dependent instructions, which the issuing and epilogue threads would pay
// on every tile or block.
struct TileCursor {
  int bh, qt, gq, img;
  __device__ __forceinline__ void init(int T, int ntq, int G, int kvh0) {
    bh = T / ntq;
    qt = T - bh * ntq;
    gq = bh % G;
    img = bh / G - kvh0;
  }
  __device__ __forceinline__ void step(int by, int ntq, int G) {
    qt += by;
    while (qt >= ntq) {
      qt -= ntq;
      ++bh;
      if (++gq == G) {
        gq = 0;
        ++img;
      }
    }
  }
};

template <int D>
struct QueryCfg {
  // warp 0 TMA producer, warps 1-2 MMA issuers (one per warpgroup), warp 3 state images,
  // warps 4-11 two epilogue warpgroups on alternate tiles
  static constexpr int THREADS = 384;
  static constexpr int EPI0 = 4;
  // registers after setmaxnreg: producer / MMA / image warpgroup, epilogue warpgroups (the
  // epilogue holds a 128-feature block of U in registers)
  static constexpr int R_LOW = 72, R_HIGH = 216;
  static_assert(128 * R_LOW + 256 * R_HIGH <= 384 * 168, "register split");
  static constexpr int FB = 128;                     // features per block (MMA1 N, MMA2 K)
  static constexpr int MMAX = D == 64 ? 512 : 256;   // features held in shared memory
  static constexpr int QTILE = 128 * D * 2;
  static constexpr int SP = D * 128 * (MMAX / 64) + 8 * MMAX;  // fp16 image, exponents, fp32 normaliser column
  // TMEM columns: warpgroup w owns U at w * TSTRIDE (phi' as fp16 pairs over its first FB / 2
  // columns once U is read), then O
  static constexpr int TSTRIDE = FB + D;
  static_assert(2 * TSTRIDE <= 512, "TMEM budget");
  // shared memory
  static constexpr int S_W = 0;                          // W' fp16, [D/64 regions][MMAX rows][128 B]
  static constexpr int S_SP = S_W + MMAX * 128 * (D / 64);
  static constexpr int S_Q = S_SP + SP;                  // Q stage w belongs to warpgroup w
  // output staging, 32 rows x 64 columns per epilogue warp: a slot of its own at d = 64; at
  // d = 128 (no room for eight) one slot per TMEM lane quarter, shared by the two warpgroups'
  // warps of that quarter in tile order
  static constexpr bool OWN_SLOT = D == 64;
  static constexpr int NSLOT = OWN_SLOT ? 8 : 4;
  static constexpr int S_STG = S_Q + 2 * QTILE;
  static constexpr int S_BAR = S_STG + NSLOT * 32 * 128;
  // PHI in halves per warpgroup (2 w + h): phi' of features 64 h .. 64 h + 63 of the block
  static constexpr int B_QF = 0, B_QE = 2, B_CVT = 4, B_UF = 6, B_PHI = 8, B_M2 = 12, B_OF = 14, B_OE = 16,
                       B_SF = 18, B_SE = 19, B_STG = 20, NBAR = 24;
  static constexpr int S_TPTR = S_BAR + NBAR * 8;
  static constexpr int S_ABORT = S_TPTR + 8;
  static constexpr int S_IMGS = S_ABORT + 4;  // state images loaded so far (published by warp 3)
  static constexpr int SMEM = S_ABORT + 16 + 1024;
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(S_SP % 1024 == 0 && S_Q % 1024 == 0 && S_STG % 1024 == 0, "128-byte swizzled operands start on 1024-byte boundaries");
};

// Query pass.  The CTA's tiles go alternately to two epilogue warpgroups, each with its own
// U and O buffers in tensor memory, its own Q stage and its own MMA-issuing thread, so one
// warpgroup's exponentials run while the tensor cores serve the other's contraction and next
// projection.  Blocks are 128 features wide (at d = 128 a 128-wide projection costs the tensor
// pipe as many cycles per MMA as a 64-wide one, so the wider block halves the projection MMAs);
// phi' goes as fp16 pairs over the first half of the block's own U columns, and the next
// projection is issued right behind the contraction that reads them (one thread's MMAs execute
// in issue order), so U's arrival also means the previous contraction has completed.  The row
// stabiliser is raised lazily across blocks with an exact rescale of O and of the normaliser,
// which the epilogue sums itself (phi' times the state's fp32 normaliser column).  The
// projection runs in fp16: each warpgroup rewrites its next Q tile in place as fp16 times 2^-k,
// one k per row that puts the row's largest |q| in [2^14, 2^15), and multiplies that row's U by
// 2^k.
template <int D>
__global__ void __launch_bounds__(QueryCfg<D>::THREADS, 1) query_pass_sm100(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO, const float* __restrict__ W,
    const unsigned char* __restrict__ op_img, int L, int m, int H, int Hkv, int ntiles_total, int op_bytes,
    float wscale) {
  using C = QueryCfg<D>;
  constexpr int NT = C::THREADS;
  constexpr int FB = C::FB;
  extern __shared__ unsigned char smem_raw[];
  griddep_launch_dependents();  // the next kernel on the stream may be scheduled as SMs free up
  // offset the __shared__ array itself (not via an integer cast), so that every pointer derived
  // from it stays a shared-memory pointer and compiles to shared loads and stores
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ntq = (L + 127) / 128;
  const int G = H / Hkv;
  const int nb = (m + FB - 1) / FB;
  const int per = ntiles_total / gridDim.x, extra = ntiles_total % gridDim.x;
  const int T0 = blockIdx.x * per + min(static_cast<int>(blockIdx.x), extra);
  const int n = per + (static_cast<int>(blockIdx.x) < extra ? 1 : 0);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::S_ABORT);
  uint32_t* tptr_slot = reinterpret_cast<uint32_t*>(smem + C::S_TPTR);
  auto bar = [&](int i) { return sbase + C::S_BAR + 8u * i; };
  // kv head of a tile (b * Hkv + h / G = (b * H + h) / G); non-decreasing along the tile order,
  // so the CTA's tiles visit each kv head once: image index 0 .. nimg - 1
  const int kvh0 = T0 / ntq / G;
  const int nimg = n > 0 ? (T0 + n - 1) / ntq / G - kvh0 + 1 : 0;
  int* img_count = reinterpret_cast<int*>(smem + C::S_IMGS);

  if (warp == 0 && lane == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(C::B_QF + i), 1);
      mbar_init(bar(C::B_QE + i), 1);
      mbar_init(bar(C::B_CVT + i), 4);  // one arrival per epilogue warp
      mbar_init(bar(C::B_UF + i), 1);
      mbar_init(bar(C::B_PHI + 2 * i), 4);
      mbar_init(bar(C::B_PHI + 2 * i + 1), 4);
      mbar_init(bar(C::B_M2 + i), 1);   // the issuer's final drain
      mbar_init(bar(C::B_OF + i), 1);
      mbar_init(bar(C::B_OE + i), 4);
    }
    mbar_init(bar(C::B_SF), 1);
    mbar_init(bar(C::B_SE), 2);  // an image is released once both issuers are done with it
    for (int i = 0; i < 4; ++i) mbar_init(bar(C::B_STG + i), 1);
    *abort_flag = 0;
    *img_count = 0;
    fence_barrier_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmO);
    // the first two Q tiles and the first image go out now, under the W' fill below
    for (int it = 0; it < min(n, 2); ++it) {
      const int T = T0 + it;
      mbar_arrive_expect_tx(bar(C::B_QF + it), C::QTILE);
#pragma unroll
      for (int r = 0; r < D / 64; ++r)
        tma_load_3d(sbase + C::S_Q + it * C::QTILE + r * (128 * 128), &tmQ, bar(C::B_QF + it), 64 * r, (T % ntq) * 128,
                    T / ntq);
    }
    // the state images are written by the kernel before this one on the stream
    griddep_wait();
    if (n > 0) {
      mbar_arrive_expect_tx(bar(C::B_SF), op_bytes);
      bulk_load(sbase + C::S_SP, op_img + static_cast<size_t>(kvh0) * op_bytes, op_bytes, bar(C::B_SF));
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tptr_slot), 512);
    tmem_relinquish();
  }
  // W' in fp16 as the K-major, 128B-swizzled B operand of MMA1: row f, 16-byte chunk c at c ^ (f % 8)
  {
    const int rows = nb * FB;
    constexpr int CPR = D / 8;  // 16-byte chunks per row
    for (int item = tid; item < rows * CPR; item += NT) {
      const int f = item / CPR, c = item % CPR;
      const int rg = c >> 3, cc = c & 7;  // 64-dim region, chunk within the 128-byte row
      uint32_t h[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float w0 = 0.f, w1 = 0.f;
        if (f < m) {
          const float2 v = *reinterpret_cast<const float2*>(W + static_cast<size_t>(f) * D + 8 * c + 2 * k);
          w0 = v.x * wscale;
          w1 = v.y * wscale;
        }
        h[k] = pack_f16x2(w0, w1);
      }
      const int off = rg * (C::MMAX * 128) + f * 128 + ((cc ^ (f & 7)) << 4);
      *reinterpret_cast<uint4*>(smem + C::S_W + off) = make_uint4(h[0], h[1], h[2], h[3]);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tptr_slot;
  unsigned int* err = &g_sm100_error_word;
  // registers: the producer / MMA warpgroup gives part of its share to the two epilogue
  // warpgroups (128 x R_LOW + 256 x R_HIGH <= 384 x 168, the launch allocation; the host checks
  // the compiled count before launching)
  if (warp < C::EPI0) {
  setmaxnreg_dec<C::R_LOW>();
  if (warp == 0) {
    // ---------------- producer: Q tiles (stage = tile parity) ----------------
    if (lane == 0) {
      int issued = 0;  // tiles 0 and 1 were issued during the set-up
      TileCursor pc;
      pc.init(T0, ntq, G, kvh0);
      for (int it = 0; it < n; ++it, pc.step(1, ntq, G)) {
        const int s = it & 1;
        if (it >= 2) {
          if (!mbar_wait<true>(bar(C::B_QE + s), ((it >> 1) - 1) & 1, abort_flag, err)) break;
          mbar_arrive_expect_tx(bar(C::B_QF + s), C::QTILE);
#pragma unroll
          for (int r = 0; r < D / 64; ++r)
            tma_load_3d(sbase + C::S_Q + s * C::QTILE + r * (128 * 128), &tmQ, bar(C::B_QF + s), 64 * r, pc.qt * 128,
                        pc.bh);
        }
        issued = it + 1;
      }
      for (int it = max(0, issued - 2); it < issued; ++it)
        mbar_wait(bar(C::B_QF + (it & 1)), (it >> 1) & 1, abort_flag, err, 200000000ull);
    }
  } else if (warp == 3) {
    // ---------------- state images: image k once both issuers have released image k - 1 ----------------
    // The image warp is the only waiter on SF, so it waits its phases in order, and publishes a count
    // of loaded images: a warpgroup whose tiles skip a kv head cannot mistake an earlier phase of the
    // same parity for its image.
    if (lane == 0 && n > 0) {
      int k = 0;
      bool inflight = true;  // image 0, issued during the set-up
      for (; k < nimg; ++k) {
        if (k >= 1) {
          if (!mbar_wait<true>(bar(C::B_SE), (k - 1) & 1, abort_flag, err)) break;
          mbar_arrive_expect_tx(bar(C::B_SF), op_bytes);
          bulk_load(sbase + C::S_SP, op_img + static_cast<size_t>(kvh0 + k) * op_bytes, op_bytes, bar(C::B_SF));
          inflight = true;
        }
        if (!mbar_wait<true>(bar(C::B_SF), k & 1, abort_flag, err)) break;
        inflight = false;
        st_release_shared(img_count, k + 1);
      }
      if (inflight) mbar_wait(bar(C::B_SF), k & 1, abort_flag, err, 200000000ull);  // drain after a failure
    }
  } else if (warp == 1 || warp == 2) {
    // ---------------- MMA issuer of warpgroup w = warp - 1: its tiles w, w + 2, ... ----------------
    // Per block: the contraction once phi' is stored (and, on a tile's first block, O read out),
    // then at once the next block's projection into the same columns; across tiles that
    // projection waits for the next tile's Q, which the epilogue converts after handing over the
    // tile's last block.
    if (lane == 0) {
      const int w = warp - 1;
      const uint32_t id2 = idesc_f16(128, D, false, false);
      const uint32_t dU = tbase + w * C::TSTRIDE, dO = dU + FB;
      const uint32_t qbase = sbase + C::S_Q + w * C::QTILE;
      const int ntw = (n - w + 1) / 2;  // my tiles
      const int nblk = ntw * nb;        // my blocks
      int rel = 0;                      // images below rel released by me
      bool ok = true;
      // releases image rel without having used it (after its predecessor's release completed,
      // so that the arrival counts towards the right phase)
      auto release_unused = [&]() {
        if (rel >= 1 && !mbar_wait(bar(C::B_SE), (rel - 1) & 1, abort_flag, err)) return false;
        mbar_arrive(bar(C::B_SE));
        ++rel;
        return true;
      };
      // U = (2^-k Q) W'^T in fp16 for my block b, always FB columns wide: W' rows past m are
      // zero, so every U column the epilogue reads is written (its e = -inf masks it).  The
      // commit also covers the contraction issued before it.
      const uint32_t id1 = idesc_f16(128, FB, false, false);
      auto mma1 = [&](int j) {
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t qo = (ks >> 2) * (128 * 128) + 32 * (ks & 3);
          const uint32_t wo = (ks >> 2) * (C::MMAX * 128) + (FB * j) * 128 + 32 * (ks & 3);
          mma_ss(dU, sdesc_sw128(qbase + qo, 16, 1024), sdesc_sw128(sbase + C::S_W + wo, 16, 1024), id1,
                 ks > 0 ? 1u : 0u);
        }
        mma_commit(bar(C::B_UF + w));
        if (j == nb - 1) mma_commit(bar(C::B_QE + w));  // the Q stage may take my next tile
      };
      // before the first projection of my tile tcn: release the images that precede its image
      // and that I never used, then wait for its Q to be converted
      auto enter_tile = [&](int tcn, int kn) {
        while (rel < kn)
          if (!release_unused()) return false;
        return mbar_wait(bar(C::B_CVT + w), tcn & 1, abort_flag, err);
      };
      TileCursor cur;  // my tile t = w + 2 * tc
      if (nblk > 0) {
        cur.init(T0 + w, ntq, G, kvh0);
        ok = enter_tile(0, cur.img);
        if (ok) {
          tc_fence_after();
          mma1(0);
        }
      }
      for (int b = 0, tc = 0, j = 0; b < nblk && ok; ++b) {
        const int t = w + 2 * tc, k = cur.img;
        const bool more = b + 1 < nblk, boundary = (j == nb - 1);
        if (j == 0) {
          if (tc >= 1 && !mbar_wait(bar(C::B_OE + w), (tc - 1) & 1, abort_flag, err)) break;
          if (!wait_count_above(img_count, k, abort_flag, err)) break;
        }
        const int bw = min(FB, m - FB * j);
        bool phi_ok = true;
        for (int h = 0; h < 2 && phi_ok; ++h) {  // MMA2: O += phi' S', each half once its phi' is stored
          if (!(phi_ok = mbar_wait(bar(C::B_PHI + 2 * w + h), b & 1, abort_flag, err))) break;
          tc_fence_after();
          for (int ks = 4 * h; ks < min(4 * h + 4, bw / 16); ++ks) {  // 16 features per step, two per TMEM column
            const int fk = FB * j + 16 * ks;
            const uint64_t bd = sdesc_sw128(sbase + C::S_SP + (fk >> 6) * (D * 128) + 32 * ((fk & 63) >> 4), 16, 1024);
            mma_ts(dO, dU + 8 * ks, bd, id2, (j > 0 || ks > 0) ? 1u : 0u);
          }
        }
        if (!phi_ok) break;
        if (boundary) {
          mma_commit(bar(C::B_OF + w));
          TileCursor nx = cur;  // my next tile, t + 2
          nx.step(2, ntq, G);
          const int knext = t + 2 < n ? nx.img : nimg;
          if (knext > k && k < nimg - 1) {  // done with image k: released when these MMAs complete
            mma_commit(bar(C::B_SE));
            rel = k + 1;
          }
          if (more) {  // first block of my next tile, once its Q is converted
            if (!enter_tile(tc + 1, nx.img)) break;
            tc_fence_after();
            mma1(0);
          }
          cur = nx;
          ++tc;
          j = 0;
        } else {
          mma1(j + 1);  // behind the contraction that reads phi' from the same columns
          ++j;
        }
      }
      while (ok && rel < nimg - 1) ok = release_unused();
      if (nblk >= 1) {  // everything I issued has completed
        mma_commit(bar(C::B_M2 + w));
        mbar_wait(bar(C::B_M2 + w), 0, abort_flag, err, 200000000ull);
      }
    }
  }
  } else {
    setmaxnreg_inc<C::R_HIGH>();
    // ---------------- epilogue warpgroup ewg: tiles ewg, ewg + 2, ... ----------------
    const int eq = warp & 3;
    const int ewg = (warp - C::EPI0) >> 2;
    const int r = eq * 32 + lane;  // query row within the tile (TMEM lane)
    const uint32_t cU = ewg * C::TSTRIDE, cO = cU + FB;  // TMEM columns: U, then phi' over it; O
    // the image holds [atoms][D rows][64 features] fp16, then e and the normaliser column (fp32,
    // same scaling as the image), each over m rounded up to 128 features, e = -inf past m
    const int atoms = (m + 63) / 64, tail = (m + 127) / 128 * 128;
    const float* ev = reinterpret_cast<const float*>(smem + C::S_SP + D * 128 * atoms);
    const float* sd = ev + tail;
    // rewrites row r of Q tile t (Q stage ewg) as fp16 x 2^-k and returns 2^k; k = 0 unless the
    // row's largest |q| reaches 2^15, when it brings it into [2^14, 2^15) so that no entry
    // overflows fp16.  Thread r starts at chunk r % 8 so that the eight threads of a
    // shared-memory wavefront hit different banks.
    auto prepare = [&](int tcount) -> float {
      mbar_wait(bar(C::B_QF + ewg), tcount & 1, abort_flag, err);
      unsigned char* qrow = smem + C::S_Q + ewg * C::QTILE + r * 128;
      uint4 v[D / 8];
      uint32_t emax = 0;
#pragma unroll
      for (int rg = 0; rg < D / 64; ++rg)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          v[8 * rg + c] = *reinterpret_cast<const uint4*>(qrow + rg * (128 * 128) + 16 * (c ^ (r & 7)));
          const uint32_t wv[4] = {v[8 * rg + c].x, v[8 * rg + c].y, v[8 * rg + c].z, v[8 * rg + c].w};
#pragma unroll
          for (int k = 0; k < 4; ++k) emax = __vmaxu2(emax, wv[k] & 0x7FFF7FFFu);  // |q| of both halves
        }
      // the biased bf16 exponent of the row's largest |q|
      const int ebits = static_cast<int>(max(emax & 0xFFFFu, emax >> 16) >> 7);
      const int k = min(100, max(0, ebits - 141));
      const bool plain = __all_sync(0xffffffffu, k == 0);
      const float down = __int_as_float((127 - k) << 23);
#pragma unroll
      for (int rg = 0; rg < D / 64; ++rg)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t wv[4] = {v[8 * rg + c].x, v[8 * rg + c].y, v[8 * rg + c].z, v[8 * rg + c].w};
          uint32_t o[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float lo = __uint_as_float(wv[q] << 16), hi = __uint_as_float(wv[q] & 0xFFFF0000u);
            if (!plain) {
              lo *= down;
              hi *= down;
            }
            o[q] = pack_f16x2(lo, hi);
          }
          *reinterpret_cast<uint4*>(qrow + rg * (128 * 128) + 16 * (c ^ (r & 7))) = make_uint4(o[0], o[1], o[2], o[3]);
        }
      fence_proxy_async_smem();  // the converted tile is read by the tensor cores
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_CVT + ewg));  // this warp's 32 rows are ready
      return __int_as_float((127 + k) << 23);
    };
    float up_next = ewg < n ? prepare(0) : 1.f;
    int cntb = 0, tc = 0;
    TileCursor ec;  // my tile t
    if (ewg < n) ec.init(T0 + ewg, ntq, G, kvh0);
    for (int t = ewg; t < n; t += 2, ++tc, ec.step(2, ntq, G)) {
      const float up = up_next;
      wait_count_above(img_count, ec.img, abort_flag, err);  // this tile's image (exponents) is in
      float c = 0.f, den = 0.f;
      for (int j = 0; j < nb; ++j, ++cntb) {
        // U of this block; its arrival also means the previous block's contraction has completed
        mbar_wait(bar(C::B_UF + ewg), cntb & 1, abort_flag, err);
        tc_fence_after();
        float v[FB];
#pragma unroll
        for (int q4 = 0; q4 < FB / 32; ++q4) tmem_ld32(taddr(tbase, eq, cU + 32 * q4), *reinterpret_cast<uint32_t(*)[32]>(&v[32 * q4]));
        tmem_wait_ld();
        const float4* e4p = reinterpret_cast<const float4*>(ev + FB * j);
        const float4* s4p = reinterpret_cast<const float4*>(sd + FB * j);
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        const float2 up2 = make_float2(up, up);
#pragma unroll
        for (int k4 = 0; k4 < FB / 4; ++k4) {  // 2^k U + e and its row max, two features per fp32x2 operation
          const float4 e4 = e4p[k4];
          const float2 v01 = __ffma2_rn(make_float2(v[4 * k4 + 0], v[4 * k4 + 1]), up2, make_float2(e4.x, e4.y));
          const float2 v23 = __ffma2_rn(make_float2(v[4 * k4 + 2], v[4 * k4 + 3]), up2, make_float2(e4.z, e4.w));
          v[4 * k4 + 0] = v01.x;  // a feature past m has W' = 0 and e = -inf: v = -inf
          v[4 * k4 + 1] = v01.y;
          v[4 * k4 + 2] = v23.x;
          v[4 * k4 + 3] = v23.y;
          m4[k4 & 3] = max3(m4[k4 & 3], v[4 * k4 + 0], v[4 * k4 + 1]);
          m4[k4 & 3] = max3(m4[k4 & 3], v[4 * k4 + 2], v[4 * k4 + 3]);
        }
        const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        const bool need = (j > 0) && (mx > c + kTau);
        if (j == 0) c = mx;
        if (__any_sync(0xffffffffu, need)) {  // raise the stabiliser of the rows that need it
          const float f = need ? ex2(c - mx) : 1.f;
          scale_tmem_row(taddr(tbase, eq, cO), D / 8, f);
          den *= f;
        }
        if (need) c = mx;
        // phi' = 2^(2^k U + e - c) as fp16 pairs over U's first columns; normaliser in fp32
        const float2 nc2 = make_float2(-c, -c);
        float2 den2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int q4 = 0; q4 < FB / 32; ++q4) {
          uint32_t ph[16];
#pragma unroll
          for (int k4 = 0; k4 < 8; ++k4) {
            const float4 s4 = s4p[8 * q4 + k4];
            const float* a = &v[32 * q4 + 4 * k4];
            const float2 b01 = __fadd2_rn(make_float2(a[0], a[1]), nc2), b23 = __fadd2_rn(make_float2(a[2], a[3]), nc2);
            const float2 p01 = make_float2(ex2(b01.x), ex2(b01.y)), p23 = make_float2(ex2(b23.x), ex2(b23.y));
            den2 = __ffma2_rn(p01, make_float2(s4.x, s4.y), den2);
            den2 = __ffma2_rn(p23, make_float2(s4.z, s4.w), den2);
            ph[2 * k4] = pack_f16x2(p01.x, p01.y);
            ph[2 * k4 + 1] = pack_f16x2(p23.x, p23.y);
          }
          tmem_st16(taddr(tbase, eq, cU + 16 * q4), ph);
          if (q4 & 1) {  // this half's phi' is stored: its contraction steps may go
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_PHI + 2 * ewg + (q4 >> 1)));
          }
        }
        den += den2.x + den2.y;
      }
      // the tile's blocks are handed over: convert the next tile's Q while the last MMA2 runs
      if (t + 2 < n) up_next = prepare(tc + 1);
      // out = O / den -> bf16 -> shared staging (taken in tile order) -> TMA store
      mbar_wait(bar(C::B_OF + ewg), tc & 1, abort_flag, err);
      tc_fence_after();
      const float inv = 1.f / den;
      unsigned char* slot = smem + C::S_STG + ((C::OWN_SLOT ? 4 * ewg : 0) + eq) * (32 * 128);
      if constexpr (C::OWN_SLOT) {  // this warp's previous store has read its slot
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
      } else {  // the slot is free once the same quarter of tile t - 1 has been stored
        if (t >= 1) mbar_wait(bar(C::B_STG + eq), (t - 1) & 1, abort_flag, err);
      }
#pragma unroll
      for (int rg = 0; rg < D / 64; ++rg) {
        if (rg > 0) {  // the previous region's store has read the slot
          if (lane == 0) bulk_wait_read<0>();
          __syncwarp();
        }
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t t32[32];
          tmem_ld32(taddr(tbase, eq, cO + 64 * rg + 32 * h2), t32);
          tmem_wait_ld();
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            uint32_t w4[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
              w4[k] = pack_bf16x2(__uint_as_float(t32[8 * c4 + 2 * k]) * inv,
                                  __uint_as_float(t32[8 * c4 + 2 * k + 1]) * inv);
            const int c8 = 4 * h2 + c4;
            *reinterpret_cast<uint4*>(slot + lane * 128 + ((c8 ^ (lane & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
        if (rg == D / 64 - 1) {  // this warp has read all of its O rows: the next tile may accumulate
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(C::B_OE + ewg));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tmO, smem_u32(slot), 64 * rg, ec.qt * 128 + 32 * eq, ec.bh);
          bulk_commit();
        }
      }
      if (!C::OWN_SLOT && lane == 0) {
        bulk_wait_read<0>();
        mbar_arrive(bar(C::B_STG + eq));  // the slot is free for tile t + 1
      }
    }
    if (lane == 0) bulk_wait<0>();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, 512);
}

#include "query_pass_d64.cuh"

// ============================================================================
// Host side
// ============================================================================
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [heads, L, d] bf16, boxes of 64 dims x 128 rows x 1 head, 128-byte swizzle; rows past L read as zero
// and are not written.
int make_map(CUtensorMap* map, const void* base, int d, int L, int heads, int box_rows = 128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return set_error(FAVOR_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(L) * d * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_errorf(FAVOR_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return FAVOR_OK;
}

int num_sms() {
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 1;
}

// The kernels that rebalance registers between warpgroups (setmaxnreg) need the launch to
// hold at least what the rebalanced warpgroups ask for, or the increase would never be
// granted: check the compiled register count once per kernel before the first launch.
int check_register_split(const void* kern, int threads, long need = -1) {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "sm100 kernel attributes: %s", cudaGetErrorString(e));
  const long have = static_cast<long>(fa.numRegs) * threads;
  if (need < 0) need = 128L * kRegsLow + static_cast<long>(threads - 128) * kRegsHigh;
  if (have < need)
    return set_errorf(FAVOR_ERR_UNSUPPORTED, "sm100 kernel compiled with %d registers per thread: %ld < %ld needed",
                      fa.numRegs, have, need);
  return FAVOR_OK;
}

template <int D>
int launch_key(const void* K, const void* V, const float* W, void* partials, const Plan& p, cudaStream_t st,
               bool overlap, bool relu = false) {
  CUtensorMap mk, mv;
  const int heads = p.B * p.Hkv;
  int rc = make_map(&mk, K, D, p.L, heads);
  if (rc == FAVOR_OK) rc = make_map(&mv, V, D, p.L, heads);
  if (rc != FAVOR_OK) return rc;
  // d = 64: the two-warpgroup kernel (256 features per CTA when m > 128); d = 128: the lock-step kernel
  void (*kern)(const CUtensorMap, const CUtensorMap, const float*, float*, float*, int, int, int, int, int, float, float);
  int smem_bytes, threads;
  const int nfeat = key_features_per_cta(p.d, p.m);
  if constexpr (D == 64) {
    // each variant's register split is checked once
    static const int split[4] = {
        check_register_split(reinterpret_cast<const void*>(key_pass_pp_sm100<false, false>), KeyPP<false>::THREADS),
        check_register_split(reinterpret_cast<const void*>(key_pass_pp_sm100<true, false>), KeyPP<true>::THREADS),
        check_register_split(reinterpret_cast<const void*>(key_pass_pp_sm100<false, true>), KeyPP<false>::THREADS),
        check_register_split(reinterpret_cast<const void*>(key_pass_pp_sm100<true, true>), KeyPP<true>::THREADS)};
    const bool wide = nfeat == 256;
    kern = wide ? (relu ? key_pass_pp_sm100<true, true> : key_pass_pp_sm100<true, false>)
                : (relu ? key_pass_pp_sm100<false, true> : key_pass_pp_sm100<false, false>);
    smem_bytes = wide ? KeyPP<true>::SMEM : KeyPP<false>::SMEM;
    threads = KeyPP<true>::THREADS;
    const int v = (relu ? 2 : 0) + (wide ? 1 : 0);
    if (split[v] != FAVOR_OK)
      return check_register_split(reinterpret_cast<const void*>(kern), threads);
  } else {
    if (relu) return set_error(FAVOR_ERR_UNSUPPORTED, "sm100 key pass: the ReLU map needs d = 64");
    kern = key_pass_sm100<D>;
    smem_bytes = KeyCfg<D>::SMEM;
    threads = kThreads;
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "sm100 key pass attribute: %s", cudaGetErrorString(e));
  char* base = static_cast<char*>(partials);
  dim3 grid((p.m + nfeat - 1) / nfeat, p.P, heads);
  e = launch_overlapped(kern, grid, dim3(threads), smem_bytes, st, overlap, mk, mv, W,
                        reinterpret_cast<float*>(base + p.part_S_off), reinterpret_cast<float*>(base + p.part_c_off),
                        p.L, p.m, p.P, p.chunk, p.nsb, relu ? relu_wscale(p.d) : p.wscale, p.nscale);
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "sm100 key pass launch: %s", cudaGetErrorString(e));
  return FAVOR_OK;
}

template <int D>
int launch_query(const void* Q, const float* W, const void* state, void* out, const Plan& p, cudaStream_t st,
                 bool overlap) {
  using C = QueryCfg<D>;
  CUtensorMap mq, mo;
  const int bh = p.B * p.H;
  int rc = make_map(&mq, Q, D, p.L, bh);
  if (rc == FAVOR_OK) rc = make_map(&mo, out, D, p.L, bh, 32);  // stored by each epilogue warp, 32 rows
  if (rc != FAVOR_OK) return rc;
  auto kern = query_pass_sm100<D>;
  const long need = 128L * C::R_LOW + 256L * C::R_HIGH;
  static const int split_ok = check_register_split(reinterpret_cast<const void*>(kern), C::THREADS, need);
  if (split_ok != FAVOR_OK) return check_register_split(reinterpret_cast<const void*>(kern), C::THREADS, need);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "sm100 query pass attribute: %s", cudaGetErrorString(e));
  const int ntiles = bh * ((p.L + 127) / 128);
  const int grid = ntiles < num_sms() ? ntiles : num_sms();
  const unsigned char* img = static_cast<const unsigned char*>(state) + p.st_op_off;
  e = launch_overlapped(kern, dim3(grid), dim3(C::THREADS), C::SMEM, st, overlap, mq, mo, W, img, p.L, p.m, p.H, p.Hkv,
                        ntiles, static_cast<int>(p.op_bytes), p.wscale);
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "sm100 query pass launch: %s", cudaGetErrorString(e));
  return FAVOR_OK;
}

// img: the state images of the plan's kv heads; W: m rows of d floats, w_row floats apart (cpk > 0:
// one W per kv head, w_head floats apart, and cpk CTAs per kv head)
int launch_query_d64_img(const void* Q, const float* W, int w_row, float wscale, const unsigned char* img, void* out,
                         const Plan& p, cudaStream_t st, bool overlap, bool relu, long w_head = 0, int cpk = 0) {
  using C = QueryD64;
  CUtensorMap mq, mo;
  const int bh = p.B * p.H;
  int rc = make_map(&mq, Q, C::D, p.L, bh);
  if (rc == FAVOR_OK) rc = make_map(&mo, out, C::D, p.L, bh, 32);  // stored by each output warp, 32 rows
  if (rc != FAVOR_OK) return rc;
  if (p.op_rows != C::NROWS) return set_error(FAVOR_ERR_UNSUPPORTED, "query pass: state image without the normaliser rows");
  auto kern = relu ? query_pass_d64_sm100<true> : query_pass_d64_sm100<false>;
  const long need = 128L * C::R_CTL + 128L * C::R_CVT + 256L * C::R_EPI;
  static const int split_ok[2] = {
      check_register_split(reinterpret_cast<const void*>(query_pass_d64_sm100<false>), C::THREADS, need),
      check_register_split(reinterpret_cast<const void*>(query_pass_d64_sm100<true>), C::THREADS, need)};
  if (split_ok[relu ? 1 : 0] != FAVOR_OK)
    return check_register_split(reinterpret_cast<const void*>(kern), C::THREADS, need);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "sm100 query pass attribute: %s", cudaGetErrorString(e));
  const int ntiles = bh * ((p.L + 127) / 128);
  const int grid = cpk > 0 ? p.B * p.Hkv * cpk : (ntiles < num_sms() ? ntiles : num_sms());
  e = launch_overlapped(kern, dim3(grid), dim3(C::THREADS), C::SMEM, st, overlap, mq, mo, W, img, p.L, p.m, p.H,
                        p.Hkv, ntiles, static_cast<int>(p.op_bytes), wscale, w_row, w_head, cpk);
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "sm100 query pass launch: %s", cudaGetErrorString(e));
  return FAVOR_OK;
}

// E, F: [kp][L] fp32; split: scratch of linformer_split_bytes; partials: the plan's (B = 2 B' batches)
int launch_linformer_proj(const void* K, const void* V, const float* E, const float* F, void* split, void* partials,
                          const Plan& pk, int heads, cudaStream_t st) {
  using C = LinProj;
  const int kpad = (pk.m + 127) / 128 * 128, Lpad = (pk.L + 63) / 64 * 64;
  const int threads = 256, blocks = 4 * num_sms();
  split_hi_lo_kernel<<<blocks, threads, 0, st>>>(E, F, static_cast<__nv_bfloat16*>(split), pk.m, kpad, pk.L, Lpad);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "projection split launch: %s", cudaGetErrorString(e));
  CUtensorMap mef, mk, mv;
  int rc = make_map(&mef, split, Lpad, kpad, 4);  // [4][kpad][Lpad]: boxes of 128 rows x 64 tokens
  if (rc == FAVOR_OK) rc = make_map(&mk, K, C::D, pk.L, heads, C::TT);
  if (rc == FAVOR_OK) rc = make_map(&mv, V, C::D, pk.L, heads, C::TT);
  if (rc != FAVOR_OK) return rc;
  e = cudaFuncSetAttribute(linformer_proj_sm100, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "projection attribute: %s", cudaGetErrorString(e));
  char* base = static_cast<char*>(partials);
  const float kscale = static_cast<float>(1.0 / std::sqrt(std::sqrt(static_cast<double>(C::D))));
  e = launch_overlapped(linformer_proj_sm100, dim3(kpad / 128, pk.P, 2 * ((heads + C::HPC - 1) / C::HPC)),
                        dim3(C::THREADS), C::SMEM, st,
                        false, mef, mk, mv, reinterpret_cast<float*>(base + pk.part_S_off),
                        reinterpret_cast<float*>(base + pk.part_c_off), pk.L, pk.m, pk.P, pk.chunk, pk.nsb, heads,
                        kscale);
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "projection launch: %s", cudaGetErrorString(e));
  return FAVOR_OK;
}

int launch_query_d64(const void* Q, const float* W, const void* state, void* out, const Plan& p, cudaStream_t st,
                     bool overlap, bool relu = false) {
  return launch_query_d64_img(Q, W, p.d, relu ? relu_wscale(p.d) : p.wscale,
                              static_cast<const unsigned char*>(state) + p.st_op_off, out, p, st, overlap, relu);
}

}  // namespace

bool sm100_key_supported(const Plan& p) { return p.d == 64 || p.d == 128; }
// d = 64: the three-warpgroup kernel for m > 64 (m <= 64 is one feature block per tile and runs on
// the CUDA cores); d = 128: the two-warpgroup kernel for m <= 256
bool sm100_query_supported(const Plan& p) {
  return (p.d == 64 && p.m > 64 && p.m <= QueryD64::MMAX) || (p.d == 128 && p.m <= QueryCfg<128>::MMAX);
}

int sm100_key_pass(const void* K, const void* V, const float* W, void* partials, const Plan& p, cudaStream_t st,
                   bool overlap) {
  return p.d == 64 ? launch_key<64>(K, V, W, partials, p, st, overlap)
                   : launch_key<128>(K, V, W, partials, p, st, overlap);
}

size_t linformer_split_bytes(int kp, int L) { return 4ull * ((kp + 127) / 128 * 128) * ((L + 63) / 64 * 64) * 2; }

int sm100_linformer_proj(const void* K, const void* V, const float* E, const float* F, void* split, void* partials,
                         const Plan& pk, int heads, cudaStream_t st) {
  if (pk.d != 64) return set_error(FAVOR_ERR_UNSUPPORTED, "sm100 projection: needs d = 64");
  if (pk.chunk % LinProj::TT != 0) return set_error(FAVOR_ERR_UNSUPPORTED, "sm100 projection: chunk not a whole number of stages");
  return launch_linformer_proj(K, V, E, F, split, partials, pk, heads, st);
}

int sm100_linformer_query(const void* Q, const void* state, void* out, const Plan& pq, const Plan& pk, cudaStream_t st) {
  if (!(pq.d == 64 && pq.m > 64 && pq.m <= QueryD64::MMAX))
    return set_error(FAVOR_ERR_UNSUPPORTED, "sm100 projected query: needs d = 64 and 64 < k <= 512");
  // one launch: each kv head t gets its own CTAs (its W, the projected keys d^-1/4 E K, is the state
  // rows of head B Hkv + t, rows d + 1 floats apart; its projected values F V are the state image of
  // head t).  The CTAs read W before any wait, and W is the reduction's output: an ordinary launch.
  const int heads = pq.B * pq.Hkv, D1 = pq.d + 1, G = pq.H / pq.Hkv, ntq = (pq.L + 127) / 128;
  const int cpk = std::max(1, std::min(G * ntq, (num_sms() + heads / 2) / heads));
  const float* S = reinterpret_cast<const float*>(static_cast<const char*>(state) + pk.st_S_off);
  const unsigned char* img = static_cast<const unsigned char*>(state) + pk.st_op_off;
  return launch_query_d64_img(Q, S + static_cast<size_t>(heads) * pq.m * D1, D1, pq.wscale, img, out, pq, st, false,
                              false, static_cast<long>(pq.m) * D1, cpk);
}

int sm100_query_pass_relu(const void* Q, const float* W, const void* state, void* out, const Plan& p, cudaStream_t st) {
  if (!(p.d == 64 && p.m > 64 && p.m <= QueryD64::MMAX))
    return set_error(FAVOR_ERR_UNSUPPORTED, "sm100 query pass: the ReLU map needs d = 64 and 64 < m <= 512");
  return launch_query_d64(Q, W, state, out, p, st, false, true);
}

int sm100_key_pass_relu(const void* K, const void* V, const float* W, void* partials, const Plan& p, cudaStream_t st) {
  if (p.d != 64) return set_error(FAVOR_ERR_UNSUPPORTED, "sm100 key pass: the ReLU map needs d = 64");
  return launch_key<64>(K, V, W, partials, p, st, false, true);
}

int sm100_query_pass(const void* Q, const float* W, const void* state, void* out, const Plan& p, cudaStream_t st,
                     bool overlap) {
  return p.d == 64 ? launch_query_d64(Q, W, state, out, p, st, overlap)
                   : launch_query<128>(Q, W, state, out, p, st, overlap);
}

int sm100_read_and_clear_error(unsigned int* word) {
  unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(word, g_sm100_error_word, sizeof(unsigned int));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_sm100_error_word, &zero, sizeof(unsigned int));
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "reading the device error word: %s", cudaGetErrorString(e));
  return FAVOR_OK;
}

}  // namespace favor
