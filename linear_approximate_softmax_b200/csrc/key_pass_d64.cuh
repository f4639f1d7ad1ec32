// Key pass for d = 64 (included by kernels_sm100.cu).
//
// "Rethinking Attention with Performers" (Abstract; 제안 방법 / proposed method), key side:
// S_part = sum_t phi(k_t') [v_t | 1]^T over one chunk of keys, phi(k') = exp(W k' - |k'|^2/2)/sqrt(m),
// for 128 features of one kv head; in log2 units with a per-feature stabiliser c_f:
//   MMA1  U^T[f, t] = [W'_f | 1 1] . [k_t | -n_hi(k_t) -n_lo(k_t)]   fp16, A = W' (tensor memory),
//                                                                   B = the K block (converted in place)
//   exp   phi^T[f, t] = 2^(U^T[f, t] - c_f)                           bf16, over the block's own U columns
//   MMA2  S[f, :64] += phi^T[f, :] . V,  S[f, 64] += phi^T[f, :] . 1  A = phi^T (tensor memory)
// where n(k) = d^-1/2 log2(e) |k|^2 / 2, split into two fp16 parts so that the projection itself
// subtracts it.  One CTA per (128-feature group, key chunk, kv head); 16 warps:
//   warp 0       TMA producer: K and V blocks of 64 keys into NST stages
//   warps 1, 2   MMA issuers of epilogue warpgroups 0 and 1 (alternate blocks)
//   warps 4-11   two epilogue warpgroups (one feature per thread, the block's 64 keys per row)
//   warps 12-15  converter warpgroup: each K block to fp16 in place, with the two norm columns
// Each epilogue warpgroup owns two U buffers and its S accumulator in tensor memory: blocks
// alternate between the buffers, phi is written over the block's own U columns, and a buffer is
// projected into again (two blocks later) once the contraction that read it has completed, so
// the exponential loop never waits for a contraction.
//
// Stabiliser: c_f is the exact maximum of the warpgroup's first block for feature f; later blocks
// exponentiate with it in one pass and redo the block (raising c_f, rescaling the feature's S row
// exactly) only if their maximum exceeds c_f + 64: phi <= 2^64 keeps bf16 and the fp32 state finite.
// The two accumulators are merged exactly at the end: S = 2^(c0 - c) S0 + 2^(c1 - c) S1.
//
// Keys whose elements reach 2^15 (fp16 range) or whose norm term exceeds 3 * 10^4 make their block
// a slow block: the converter scales such a key by 2^-s and leaves the norm columns zero, and the
// epilogue applies 2^s and subtracts the exact fp32 norm itself.
struct KeyD64 {
  static constexpr int D = 64;
  static constexpr int THREADS = 512;
  static constexpr int EPI0 = 4, CVT0 = 12;
  static constexpr int TB = 64;            // keys per block
  static constexpr int NST = 6;            // K / V stages
  static constexpr int KB = TB * 128;      // one K (or V) block: 64 rows of 128 B
  static constexpr float kRaise = 64.f;    // phi <= 2^64
  // tensor memory: W' fp16 pairs (32 columns) and the norm columns [1 1 0 ...] (8); warpgroup w at
  // 48 + 208 w: two U buffers of 64 columns, then S (64 outputs, the normaliser, 15)
  static constexpr int T_W = 0, T_WX = 32, T_WG0 = 48, T_WGS = 208, T_U = 0, T_S = 128;
  // shared memory (1024-aligned base)
  static constexpr int S_K = 0;                     // NST K blocks (fp16 after conversion), SW128
  static constexpr int S_KX = S_K + NST * KB;       // NST norm-column atoms (only chunks 0-1 per row)
  static constexpr int S_V = S_KX + NST * KB;       // NST V blocks (bf16), SW128
  static constexpr int S_ONES = S_V + NST * KB;     // [16 rows x 64 keys] bf16, row 0 = 1
  static constexpr int S_NRM = S_ONES + 2048;       // per stage: n(k) [64] and 2^s [64] (slow blocks)
  static constexpr int S_SLOW = S_NRM + NST * 512;  // per stage: one flag per converter warp
  static constexpr int S_CW = S_SLOW + NST * 16;    // end: stabilisers of the two accumulators [2][128]
  static constexpr int S_BAR = S_CW + 1024;
  static constexpr int B_KVF = 0, B_KVE = NST, B_CVF = 2 * NST, B_UF = 3 * NST, B_PHI = B_UF + 4, B_M2 = B_PHI + 4,
                       NBAR = B_M2 + 4;
  static constexpr int S_TPTR = S_BAR + NBAR * 8;
  static constexpr int S_ABORT = S_TPTR + 8;
  static constexpr int SMEM = S_ABORT + 16 + 1024;
  static constexpr int R_CTL = 80, R_CVT = 80, R_EPI = 176;
  static_assert(128 * R_CTL + 128 * R_CVT + 256 * R_EPI <= 65536, "register split");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(S_KX % 1024 == 0 && S_V % 1024 == 0 && S_ONES % 1024 == 0, "swizzled operands on 1024-byte boundaries");
};

__global__ void __launch_bounds__(KeyD64::THREADS, 1) key_pass_d64_sm100(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const float* __restrict__ W,
    float* __restrict__ part_S, float* __restrict__ part_c, int L, int m, int P, int chunk, int nsb, float wscale,
    float nscale) {
  using C = KeyD64;
  constexpr int D = C::D, NST = C::NST;
  extern __shared__ unsigned char smem_raw[];
  griddep_launch_dependents();  // the next kernel on the stream may be scheduled as SMs free up
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = blockIdx.x, p = blockIdx.y, head = blockIdx.z;
  const int f0 = grp * 128, gw = min(128, m - f0);
  const int t_begin = p * chunk, t_end = min(L, t_begin + chunk);
  const int nblk = (t_end - t_begin + C::TB - 1) / C::TB;  // >= 1
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::S_ABORT);
  uint32_t* tptr_slot = reinterpret_cast<uint32_t*>(smem + C::S_TPTR);
  auto bar = [&](int i) { return sbase + C::S_BAR + 8u * i; };

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar(C::B_KVF + s), 1);
      mbar_init(bar(C::B_KVE + s), 1);
      mbar_init(bar(C::B_CVF + s), 4);  // one arrival per converter warp
    }
    for (int x = 0; x < 4; ++x) {
      mbar_init(bar(C::B_UF + x), 1);
      mbar_init(bar(C::B_PHI + x), 4);  // one arrival per epilogue warp
      mbar_init(bar(C::B_M2 + x), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    // the first stages' loads go out now, under the set-up below
    for (int i = 0; i < min(nblk, NST); ++i) {
      mbar_arrive_expect_tx(bar(C::B_KVF + i), 2 * C::KB);
      tma_load_3d(sbase + C::S_K + i * C::KB, &tmK, bar(C::B_KVF + i), 0, t_begin + C::TB * i, head);
      tma_load_3d(sbase + C::S_V + i * C::KB, &tmV, bar(C::B_KVF + i), 0, t_begin + C::TB * i, head);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tptr_slot), 512);
    tmem_relinquish();
  }
  // ones tile: K-major [16 rows x 64 keys], row 0 = 1.0 (bf16), rows 1..15 = 0
  for (int i = tid; i < 2048 / 4; i += C::THREADS)
    reinterpret_cast<uint32_t*>(smem + C::S_ONES)[i] = (i < 32) ? 0x3F803F80u : 0u;
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tptr_slot;
  unsigned int* err = &g_sm100_error_word;
  float* cw = reinterpret_cast<float*>(smem + C::S_CW);

  if (warp >= C::CVT0) {
    // W' (fp16 pairs) and the norm columns into tensor memory as the A operand of MMA1: lane = feature
    const int frow = (warp & 3) * 32 + lane;
    uint32_t wr[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float w0 = 0.f, w1 = 0.f;
      if (frow < gw) {
        const float2 v = *reinterpret_cast<const float2*>(W + static_cast<size_t>(f0 + frow) * D + 2 * j);
        w0 = v.x * wscale;
        w1 = v.y * wscale;
      }
      wr[j] = pack_f16x2(w0, w1);
    }
    tmem_st32(taddr(tbase, warp & 3, C::T_W), wr);
    uint32_t wx[8] = {0x3C003C00u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};  // fp16 (1, 1): K columns 64 and 65
    tmem_st8(taddr(tbase, warp & 3, C::T_WX), wx);
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp < C::EPI0) {
    setmaxnreg_dec<C::R_CTL>();
    if (warp == 0) {
      // ---------------- TMA producer: block i into stage i % NST ----------------
      if (lane == 0) {
        int issued = min(nblk, NST);
        for (int i = NST; i < nblk; ++i) {
          const int s = i % NST;
          if (!mbar_wait<true>(bar(C::B_KVE + s), ((i / NST) - 1) & 1, abort_flag, err)) break;
          mbar_arrive_expect_tx(bar(C::B_KVF + s), 2 * C::KB);
          tma_load_3d(sbase + C::S_K + s * C::KB, &tmK, bar(C::B_KVF + s), 0, t_begin + C::TB * i, head);
          tma_load_3d(sbase + C::S_V + s * C::KB, &tmV, bar(C::B_KVF + s), 0, t_begin + C::TB * i, head);
          issued = i + 1;
        }
        for (int i = max(0, issued - NST); i < issued; ++i)
          mbar_wait(bar(C::B_KVF + i % NST), (i / NST) & 1, abort_flag, err, 200000000ull);
      }
    } else if (warp == 1 || warp == 2) {
      // ---------------- MMA issuer of warpgroup w: blocks i = w, w + 2, ... (its b-th: i = 2b + w) ----------------
      if (lane == 0) {
        const int w = warp - 1;
        const uint32_t tw = tbase + C::T_WG0 + w * C::T_WGS;
        const uint32_t dU = tw + C::T_U, dS = tw + C::T_S;
        const uint32_t id1 = idesc_f16(128, C::TB, false, false);
        const uint32_t idv = idesc_bf16(128, D, false, true);  // V block as an MN-major B operand
        const uint32_t ido = idesc_bf16(128, 16, false, false);
        const int nbw = (nblk - w + 1) / 2;
        int a1 = 0;
        auto issue_mma1 = [&]() -> bool {  // U^T(a1) = [W' | 1 1] [K | -n]^T into U buffer a1 % 2
          const int i = 2 * a1 + w, s = i % NST;
          if (!mbar_wait(bar(C::B_CVF + s), (i / NST) & 1, abort_flag, err)) return false;  // converted
          if (a1 >= 2 && !mbar_wait(bar(C::B_M2 + 2 * w + (a1 & 1)), ((a1 - 2) >> 1) & 1, abort_flag, err)) return false;
          tc_fence_after();
          const uint32_t d = dU + (a1 & 1) * C::TB;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            mma_ts(d, tbase + C::T_W + 8 * ks, sdesc_sw128(sbase + C::S_K + s * C::KB + 32 * ks, 16, 1024), id1,
                   ks > 0 ? 1u : 0u);
          mma_ts(d, tbase + C::T_WX, sdesc_sw128(sbase + C::S_KX + s * C::KB, 16, 1024), id1, 1u);  // - n(k)
          mma_commit(bar(C::B_UF + 2 * w + (a1 & 1)));
          ++a1;
          return true;
        };
        bool ok = true;
        for (int k = 0; k < 2 && a1 < nbw && ok; ++k) ok = issue_mma1();
        for (int b = 0; b < nbw && ok; ++b) {
          const int i = 2 * b + w, s = i % NST;
          if (!mbar_wait(bar(C::B_PHI + 2 * w + (b & 1)), (b >> 1) & 1, abort_flag, err)) break;
          tc_fence_after();
          const uint32_t aP = dU + (b & 1) * C::TB;
#pragma unroll
          for (int ks = 0; ks < C::TB / 16; ++ks) {  // S += phi^T [V | 1], 16 keys per step
            const uint32_t acc = (b > 0 || ks > 0) ? 1u : 0u;
            mma_ts(dS, aP + 8 * ks, sdesc_sw128(sbase + C::S_V + s * C::KB + 2048 * ks, 16, 1024), idv, acc);
            mma_ts(dS + D, aP + 8 * ks, sdesc_sw128(sbase + C::S_ONES + 32 * ks, 16, 1024), ido, acc);
          }
          mma_commit(bar(C::B_M2 + 2 * w + (b & 1)));
          mma_commit(bar(C::B_KVE + s));  // the stage is free once this block's contractions completed
          if (a1 < nbw) ok = issue_mma1();  // block b + 2, into the buffer this contraction read
        }
        if (nbw >= 1) mbar_wait(bar(C::B_M2 + 2 * w + ((nbw - 1) & 1)), ((nbw - 1) >> 1) & 1, abort_flag, err, 200000000ull);
      }
    }
  } else if (warp < C::CVT0) {
    setmaxnreg_inc<C::R_EPI>();
    // ---------------- epilogue warpgroup w: one feature per thread, blocks 2b + w ----------------
    const int eq = warp & 3;
    const int w = (warp - C::EPI0) >> 2;
    const int frow = eq * 32 + lane;
    const uint32_t cU = C::T_WG0 + w * C::T_WGS + C::T_U, cS = C::T_WG0 + w * C::T_WGS + C::T_S;
    const int nbw = (nblk - w + 1) / 2;
    float c = 0.f;
    for (int b = 0; b < nbw; ++b) {
      const int i = 2 * b + w, s = i % NST;
      mbar_wait(bar(C::B_UF + 2 * w + (b & 1)), (b >> 1) & 1, abort_flag, err);
      tc_fence_after();
      const uint32_t cb = cU + (b & 1) * C::TB;
      float a[C::TB];
      tmem_ld32(taddr(tbase, eq, cb), *reinterpret_cast<uint32_t(*)[32]>(&a[0]));
      tmem_ld32(taddr(tbase, eq, cb + 32), *reinterpret_cast<uint32_t(*)[32]>(&a[32]));
      tmem_wait_ld();
      // a slow block: keys scaled by 2^-s and the norm left to the epilogue (flags of the 4 converter warps)
      mbar_wait(bar(C::B_CVF + s), (i / NST) & 1, abort_flag, err);
      const int4 sl = *reinterpret_cast<const int4*>(smem + C::S_SLOW + 16 * s);
      if (sl.x | sl.y | sl.z | sl.w) {
        const float* nr = reinterpret_cast<const float*>(smem + C::S_NRM + 512 * s);
#pragma unroll
        for (int t = 0; t < C::TB; ++t) a[t] = fmaf(a[t], nr[C::TB + t], -nr[t]);
      }
      uint32_t ph[C::TB / 2];
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      auto exponentiate = [&]() {  // phi = 2^(a - c) for the whole block, as bf16 pairs
        const float2 nc2 = make_float2(-c, -c);
#pragma unroll
        for (int k2 = 0; k2 < C::TB / 2; ++k2) {
          const float2 bb = __fadd2_rn(make_float2(a[2 * k2], a[2 * k2 + 1]), nc2);
          ph[k2] = pack_bf16x2(ex2(bb.x), ex2(bb.y));
        }
      };
      if (b == 0) {  // the warpgroup's first block: the exact maximum first
#pragma unroll
        for (int k2 = 0; k2 < C::TB / 2; ++k2) m4[k2 & 3] = fmax3(m4[k2 & 3], a[2 * k2], a[2 * k2 + 1]);
        c = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        exponentiate();
      } else {
        const float2 nc2 = make_float2(-c, -c);
#pragma unroll
        for (int k2 = 0; k2 < C::TB / 2; ++k2) {
          m4[k2 & 3] = fmax3(m4[k2 & 3], a[2 * k2], a[2 * k2 + 1]);
          const float2 bb = __fadd2_rn(make_float2(a[2 * k2], a[2 * k2 + 1]), nc2);
          ph[k2] = pack_bf16x2(ex2(bb.x), ex2(bb.y));
        }
        const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        const bool need = mx > c + C::kRaise;
        if (__any_sync(0xffffffffu, need)) {  // cold: phi would exceed 2^64 for some feature
          mbar_wait(bar(C::B_M2 + 2 * w + ((b - 1) & 1)), ((b - 1) >> 1) & 1, abort_flag, err);
          tc_fence_after();
          scale_tmem_row(taddr(tbase, eq, cS), (D + 16) / 8, need ? ex2(c - mx) : 1.f);
          if (need) c = mx;
          exponentiate();
        }
      }
      // phi^T as bf16 pairs over the first 32 columns of this block's U buffer
      tmem_st16(taddr(tbase, eq, cb), *reinterpret_cast<uint32_t(*)[16]>(&ph[0]));
      tmem_st16(taddr(tbase, eq, cb + 16), *reinterpret_cast<uint32_t(*)[16]>(&ph[16]));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_PHI + 2 * w + (b & 1)));
    }
    // merge the two accumulators row by row and write this group's partial state, once the
    // kernels before this one on the stream (which may read the partial state) have completed
    griddep_wait();
    cw[w * 128 + frow] = c;
    named_bar_sync(3, 256);
    const int n0 = (nblk + 1) / 2, n1 = nblk / 2;  // blocks of each warpgroup
    const float c0 = cw[frow], c1 = cw[128 + frow];
    const float cmax = n1 > 0 ? fmaxf(c0, c1) : c0;
    if (n0 > 0) mbar_wait(bar(C::B_M2 + 0 + ((n0 - 1) & 1)), ((n0 - 1) >> 1) & 1, abort_flag, err);
    if (n1 > 0) mbar_wait(bar(C::B_M2 + 2 + ((n1 - 1) & 1)), ((n1 - 1) >> 1) & 1, abort_flag, err);
    tc_fence_after();
    const float s0 = n0 > 0 ? ex2(c0 - cmax) : 0.f, s1 = n1 > 0 ? ex2(c1 - cmax) : 0.f;
    // through shared memory (the K stages are free: every contraction has completed) so that the
    // partial state goes out in coalesced 16-byte stores; a row stride of D + 1 floats (odd) keeps
    // the 32 rows of a warp on different banks
    float* stg = reinterpret_cast<float*>(smem + C::S_K);
    const uint32_t cS0 = C::T_WG0 + C::T_S, cS1 = C::T_WG0 + C::T_WGS + C::T_S;
#pragma unroll
    for (int cc = 0; cc < D / 16; ++cc) {  // this warpgroup's half of the columns
      const int col0 = w * (D / 2) + 8 * cc;
      uint32_t v0[8], v1[8];
      tmem_ld8(taddr(tbase, eq, cS0 + col0), v0);
      tmem_ld8(taddr(tbase, eq, cS1 + col0), v1);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 8; ++k)
        stg[frow * (D + 1) + col0 + k] =
            (n1 > 0 ? __uint_as_float(v1[k]) * s1 : 0.f) + __uint_as_float(v0[k]) * s0;
    }
    if (w == 0) {  // the normaliser column
      uint32_t z0[8], z1[8];
      tmem_ld8(taddr(tbase, eq, cS0 + D), z0);
      tmem_ld8(taddr(tbase, eq, cS1 + D), z1);
      tmem_wait_ld();
      stg[frow * (D + 1) + D] = (n1 > 0 ? __uint_as_float(z1[0]) * s1 : 0.f) + __uint_as_float(z0[0]) * s0;
      if (frow < gw) part_c[(static_cast<size_t>(head) * P + p) * nsb + f0 + frow] = cmax;
    }
    named_bar_sync(3, 256);
    // this group's rows f0 .. f0 + gw - 1 are contiguous in the partial state; gw (D + 1) is a
    // multiple of 16 floats since m and f0 are multiples of 16
    float4* outp = reinterpret_cast<float4*>(part_S + ((static_cast<size_t>(head) * P + p) * m + f0) * (D + 1));
    const float4* src = reinterpret_cast<const float4*>(stg);
    for (int k = tid - C::EPI0 * 32; k < gw * (D + 1) / 4; k += 256) outp[k] = src[k];
  } else {
    setmaxnreg_dec<C::R_CVT>();
    // ---------------- converter: each K block to fp16 in place, with the norm columns ----------------
    // Two threads per key row, 32 dimensions each; thread h = 0 of a row writes its norm columns.
    const int ct = tid - C::CVT0 * 32;
    const int t = ct >> 1, h = ct & 1;
    for (int i = 0; i < nblk; ++i) {
      const int s = i % NST;
      mbar_wait(bar(C::B_KVF + s), (i / NST) & 1, abort_flag, err);
      unsigned char* krow = smem + C::S_K + s * C::KB + t * 128;
      uint4 v[4];
      float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      uint32_t emax = 0;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        v[c4] = *reinterpret_cast<const uint4*>(krow + 16 * ((4 * h + c4) ^ (t & 7)));
        const uint32_t wv[4] = {v[c4].x, v[c4].y, v[c4].z, v[c4].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 x = make_float2(__uint_as_float(wv[e] << 16), __uint_as_float(wv[e] & 0xFFFF0000u));
          acc[e & 1] = __ffma2_rn(x, x, acc[e & 1]);
          emax = __vmaxu2(emax, wv[e] & 0x7FFF7FFFu);
        }
      }
      float nsum = (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y);
      nsum += __shfl_xor_sync(0xffffffffu, nsum, 1);
      emax = max(emax & 0xFFFFu, emax >> 16);
      emax = max(emax, __shfl_xor_sync(0xffffffffu, emax, 1));
      const bool valid = t_begin + C::TB * i + t < t_end;
      const float n = valid ? nsum * nscale : INFINITY;
      // fp16 holds the key exactly unless an element reaches 2^15: then the row is scaled by 2^-k
      const int k = min(100, max(0, static_cast<int>(emax >> 7) - 141));
      const bool slow = valid && (k > 0 || n > 30000.f);
      const float down = __int_as_float((127 - k) << 23);
      uint32_t o[16];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        const uint32_t wv[4] = {v[c4].x, v[c4].y, v[c4].z, v[c4].w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          o[4 * c4 + e] = pack_f16x2(__uint_as_float(wv[e] << 16) * down, __uint_as_float(wv[e] & 0xFFFF0000u) * down);
      }
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4)
        *reinterpret_cast<uint4*>(krow + 16 * ((4 * h + c4) ^ (t & 7))) =
            make_uint4(o[4 * c4], o[4 * c4 + 1], o[4 * c4 + 2], o[4 * c4 + 3]);
      const bool any_slow = __any_sync(0xffffffffu, slow);  // the block is slow for every row of it
      if (h == 0) {
        // norm columns: (-n_hi, -n_lo) in fp16, or (-30000, 0) past the chunk end (phi = 0), or zeros
        // in a slow block (the epilogue subtracts the exact norm)
        uint32_t x0 = 0u;
        if (!valid) {
          x0 = pack_f16x2(-30000.f, 0.f);
        } else if (!any_slow) {
          const float nh = __half2float(__float2half_rn(n));
          x0 = pack_f16x2(-nh, -(n - nh));
        }
        unsigned char* xrow = smem + C::S_KX + s * C::KB + t * 128;
        *reinterpret_cast<uint4*>(xrow + 16 * (0 ^ (t & 7))) = make_uint4(x0, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(xrow + 16 * (1 ^ (t & 7))) = make_uint4(0u, 0u, 0u, 0u);
        // what the epilogue applies in a slow block: a = 2^k U - n for the rows of a slow warp, a = U for
        // the others (their projection already holds the norm)
        float* nr = reinterpret_cast<float*>(smem + C::S_NRM + 512 * s);
        nr[t] = any_slow ? n : 0.f;                                        // n is +inf past the chunk end
        nr[C::TB + t] = any_slow ? __int_as_float((127 + k) << 23) : 1.f;  // 2^k
      }
      if (lane == 0) reinterpret_cast<int*>(smem + C::S_SLOW + 16 * s)[warp & 3] = any_slow ? 1 : 0;
      fence_proxy_async_smem();  // the converted block is read by the tensor cores
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_CVF + s));
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, 512);
}
