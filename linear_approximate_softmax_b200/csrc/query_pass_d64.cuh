// Query pass for d = 64 with m > 64 features (included by kernels_sm100.cu).
//
// "Rethinking Attention with Performers" (Abstract; 제안 방법 / proposed method), query side:
// out_q = phi(q') S[:, :d] / phi(q') S[:, d], with phi(q') = exp(W q' - |q'|^2/2) / sqrt(m).
// In log2 units with the state image of the reduction (feature f's row scaled by 2^-e_f):
//   MMA1  U[q, f]  = (2^-k_q q) . W'[f, :]          A = Q tile (fp16, tensor memory), B = W' (smem)
//   exp   phi'[q, f] = 2^(2^k_q U[q, f] + e_f - c_q)  fp16, written over the block's own U columns
//   MMA2  O[q, :]  += phi'[q, block] . S'[block, :]   B = the image block, N = 64 outputs + normaliser
//   out   = O[q, :64] / O[q, 64]
// The -|q'|^2/2 term and the 1/sqrt(m) factors are constant along a query row and cancel in
// the ratio, as does the row stabiliser c_q.
//
// One persistent CTA per SM over a contiguous range of 128-query tiles; 16 warps:
//   warp 0       TMA producer: Q tiles into NQS shared-memory stages
//   warps 1, 2   MMA issuers of epilogue warpgroups 0 and 1
//   warp 3       state images: one per kv head, loaded once both issuers have released the previous
//                one, and published through a count of loaded images
//   warps 4-11   two epilogue warpgroups on alternate tiles (exponentials)
//   warps 12-15  converter / output warpgroup: converts each Q tile to fp16 into its warpgroup's
//                tensor-memory A operand, and writes each finished tile (O / normaliser -> bf16
//                -> TMA store)
// Each epilogue warpgroup owns, in tensor memory, its Q operand, two U buffers and its O
// accumulator.  Blocks of 64 features alternate between the two U buffers; the epilogue reads a
// block's U into registers and writes phi' over the same columns, so the epilogue never waits
// for a contraction: the next block's U is already in the other buffer, and a buffer is
// re-projected (two blocks later) right after the contraction that reads it is issued.  The Q conversion
// and the output run in their own warpgroup, off the exponential loop.
//
// Stabiliser: c_q is the exact maximum of the row's first block (two passes over it); later
// blocks exponentiate with that c_q in one pass and compute their maximum alongside.  phi' <=
// 2^15 keeps fp16 finite, so a block is redone only when its maximum exceeds c_q + 15: then c_q
// is raised to it and the accumulator (outputs and normaliser) rescaled exactly.
struct QueryD64 {
  static constexpr int D = 64;
  static constexpr int THREADS = 512;
  static constexpr int EPI0 = 4;        // warps 4-7: epilogue warpgroup 0, 8-11: warpgroup 1
  static constexpr int CVT0 = 12;       // warps 12-15: converter / output warpgroup
  static constexpr int FB = 64;         // features per block (one 64-feature atom of the image)
  static constexpr int NROWS = D + 16;  // image rows: 64 outputs, the normaliser, 15 zero rows
  static constexpr int MMAX = 512;
  static constexpr int NQS = 3;         // Q tile stages in shared memory
  static constexpr int QTILE = 128 * 128;
  static constexpr float kRaise = 15.f;  // phi' <= 2^15 stays finite in fp16
  // tensor memory: warpgroup w from column 256 w: Q operand (32 columns of fp16 pairs), two U
  // buffers of 64 columns (phi' over their first 32), O (64 outputs + the normaliser + 15)
  static constexpr int T_Q = 0, T_U = 32, T_O = 160, T_WG = 256;
  // shared memory (1024-aligned base)
  static constexpr int S_W = 0;                               // W' fp16 [MMAX rows][128 B], SW128
  static constexpr int SP = NROWS * 128 * (MMAX / 64) + 8 * MMAX;  // image rows, e, s
  static constexpr int S_SP = S_W + MMAX * 128;
  static constexpr int S_Q = S_SP + SP;
  static constexpr int S_STG = S_Q + NQS * QTILE;             // output staging, 4 KB per converter warp
  static constexpr int S_UP = S_STG + 4 * 4096;               // 2^k per row: [warpgroup][tile % 4][128]
  static constexpr int S_BAR = S_UP + 2 * 4 * 128 * 4;
  // CVT: one barrier per warpgroup and tile parity, so that a waiter one tile behind the converter
  // is never two phases behind a barrier
  static constexpr int B_QF = 0, B_QE = NQS, B_CVT = 2 * NQS, B_QT = B_CVT + 4, B_UF = B_QT + 2, B_PHI = B_UF + 4,
                       B_M2 = B_PHI + 4, B_OF = B_M2 + 4, B_OE = B_OF + 2, B_SF = B_OE + 2, B_SE = B_SF + 1,
                       NBAR = B_SE + 1;
  static constexpr int S_TPTR = S_BAR + NBAR * 8;
  static constexpr int S_ABORT = S_TPTR + 8;
  static constexpr int S_IMGS = S_ABORT + 4;  // images loaded so far (published by warp 3)
  static constexpr int SMEM = S_ABORT + 16 + 1024;
  // registers after setmaxnreg: control warpgroup, converter / output warpgroup, epilogue warpgroups
  static constexpr int R_CTL = 72, R_CVT = 88, R_EPI = 176;
  static_assert(128 * R_CTL + 128 * R_CVT + 256 * R_EPI <= 65536, "register split");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(S_SP % 1024 == 0 && S_Q % 1024 == 0 && S_STG % 1024 == 0, "swizzled operands on 1024-byte boundaries");
};

// RELU: the feature map max(W'q, 0) (W' then carries no log2(e)).  The image's exponents e_f become
// factors 2^e_f once the image is in (zero past m), and phi' = max(U, 0) 2^k 2^e_f 2^-c with an
// integer row stabiliser c that keeps phi' below 2^15, raised like the exponential map's.
template <bool RELU>
__global__ void __launch_bounds__(QueryD64::THREADS, 1) query_pass_d64_sm100(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO, const float* __restrict__ W,
    const unsigned char* __restrict__ op_img, int L, int m, int H, int Hkv, int ntiles_total, int op_bytes,
    float wscale, int w_row, long w_head, int cpk) {
  using C = QueryD64;
  constexpr int NQS = C::NQS;
  extern __shared__ unsigned char smem_raw[];
  griddep_launch_dependents();  // the next kernel on the stream may be scheduled as SMs free up
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ntq = (L + 127) / 128;
  const int G = H / Hkv;
  const int nb = (m + C::FB - 1) / C::FB;  // blocks per tile (>= 2: m > 64)
  // the CTA's tiles: an even share of all of them, or (cpk > 0: a W per kv head, w_head floats
  // apart) an even share of one kv head's, so that the CTA's W is one kv head's throughout
  int T0, n;
  if (cpk > 0) {
    const int hd = static_cast<int>(blockIdx.x) / cpk, c = static_cast<int>(blockIdx.x) % cpk, tph = G * ntq;
    const int per = tph / cpk, extra = tph % cpk;
    T0 = hd * tph + c * per + min(c, extra);
    n = per + (c < extra ? 1 : 0);
    W += static_cast<size_t>(hd) * w_head;
  } else {
    const int per = ntiles_total / gridDim.x, extra = ntiles_total % gridDim.x;
    T0 = blockIdx.x * per + min(static_cast<int>(blockIdx.x), extra);
    n = per + (static_cast<int>(blockIdx.x) < extra ? 1 : 0);
  }
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::S_ABORT);
  int* img_count = reinterpret_cast<int*>(smem + C::S_IMGS);
  uint32_t* tptr_slot = reinterpret_cast<uint32_t*>(smem + C::S_TPTR);
  auto bar = [&](int i) { return sbase + C::S_BAR + 8u * i; };
  const int kvh0 = T0 / ntq / G;
  const int nimg = n > 0 ? (T0 + n - 1) / ntq / G - kvh0 + 1 : 0;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < NQS; ++s) {
      mbar_init(bar(C::B_QF + s), 1);
      mbar_init(bar(C::B_QE + s), 4);  // one arrival per converter warp
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(bar(C::B_CVT + 2 * w), 4);
      mbar_init(bar(C::B_CVT + 2 * w + 1), 4);
      mbar_init(bar(C::B_QT + w), 1);
      mbar_init(bar(C::B_OF + w), 1);
      mbar_init(bar(C::B_OE + w), 4);
      for (int x = 0; x < 2; ++x) {
        mbar_init(bar(C::B_UF + 2 * w + x), 1);
        mbar_init(bar(C::B_PHI + 2 * w + x), 4);
        mbar_init(bar(C::B_M2 + 2 * w + x), 1);
      }
    }
    mbar_init(bar(C::B_SF), 1);
    mbar_init(bar(C::B_SE), 2);  // an image is released once both issuers are done with it
    *abort_flag = 0;
    *img_count = 0;
    fence_barrier_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmO);
    // the first Q tiles go out now, under the W' fill below
    for (int it = 0; it < min(n, NQS); ++it) {
      const int T = T0 + it;
      mbar_arrive_expect_tx(bar(C::B_QF + it), C::QTILE);
      tma_load_3d(sbase + C::S_Q + it * C::QTILE, &tmQ, bar(C::B_QF + it), 0, (T % ntq) * 128, T / ntq);
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
  // W' in fp16 as the K-major, 128B-swizzled B operand of MMA1: row f, 16-byte chunk c at c ^ (f % 8);
  // rows past m are zero (their e = -inf masks them)
  for (int item = tid; item < nb * C::FB * 8; item += C::THREADS) {
    const int f = item >> 3, c = item & 7;
    uint32_t h[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float w0 = 0.f, w1 = 0.f;
      if (f < m) {  // row f of W starts at f * w_row floats (w_row >= D, possibly odd)
        const float* wr = W + static_cast<size_t>(f) * w_row + 8 * c + 2 * k;
        w0 = wr[0] * wscale;
        w1 = wr[1] * wscale;
      }
      h[k] = pack_f16x2(w0, w1);
    }
    *reinterpret_cast<uint4*>(smem + C::S_W + f * 128 + ((c ^ (f & 7)) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tptr_slot;
  unsigned int* err = &g_sm100_error_word;
  float* upv = reinterpret_cast<float*>(smem + C::S_UP);  // [w][tile % 4][row]

  if (warp < C::EPI0) {
    setmaxnreg_dec<C::R_CTL>();
    if (warp == 0) {
      // ---------------- producer: Q tiles (stage = tile % NQS) ----------------
      if (lane == 0) {
        int issued = min(n, NQS);  // issued during the set-up
        TileCursor pc;
        pc.init(T0, ntq, G, kvh0);
        for (int it = 0; it < n; ++it, pc.step(1, ntq, G)) {
          if (it >= NQS) {
            const int s = it % NQS;
            if (!mbar_wait<true>(bar(C::B_QE + s), ((it / NQS) - 1) & 1, abort_flag, err)) break;
            mbar_arrive_expect_tx(bar(C::B_QF + s), C::QTILE);
            tma_load_3d(sbase + C::S_Q + s * C::QTILE, &tmQ, bar(C::B_QF + s), 0, pc.qt * 128, pc.bh);
            issued = it + 1;
          }
        }
        for (int it = max(0, issued - NQS); it < issued; ++it)
          mbar_wait(bar(C::B_QF + it % NQS), (it / NQS) & 1, abort_flag, err, 200000000ull);
      }
    } else if (warp == 3) {
      // ---------------- state images: image k once both issuers have released image k - 1 ----------------
      if (lane == 0 && n > 0) {
        // image 0 was issued during the set-up; every later image waits for the release of the one
        // before it (the only waiter on SF, so its phases are waited in order)
        int k = 0;
        bool inflight = true;  // image 0
        for (; k < nimg; ++k) {
          if (k >= 1) {
            if (!mbar_wait<true>(bar(C::B_SE), (k - 1) & 1, abort_flag, err)) break;
            mbar_arrive_expect_tx(bar(C::B_SF), op_bytes);
            bulk_load(sbase + C::S_SP, op_img + static_cast<size_t>(kvh0 + k) * op_bytes, op_bytes, bar(C::B_SF));
            inflight = true;
          }
          if (!mbar_wait<true>(bar(C::B_SF), k & 1, abort_flag, err)) break;
          inflight = false;
          if constexpr (RELU) {  // e_f -> 2^e_f in place (the next image's copy is ordered after this)
            float* ef = reinterpret_cast<float*>(smem + C::S_SP + C::NROWS * 128 * nb);
            for (int f = 0; f < nb * C::FB; ++f) ef[f] = ex2(ef[f]);
            fence_proxy_async_smem();
          }
          st_release_shared(img_count, k + 1);
        }
        if (inflight) mbar_wait(bar(C::B_SF), k & 1, abort_flag, err, 200000000ull);  // drain after a failure
      }
    } else if (warp == 1 || warp == 2) {
      // ---------------- MMA issuer of epilogue warpgroup w: its tiles w, w + 2, ... ----------------
      // Two streams over the warpgroup's blocks a = tile * nb + j: MMA2(a) once the epilogue has
      // written phi'(a), then at once MMA1(a + 2) into the same U buffer (for a tile's first block,
      // once its Q operand is converted): the tensor core runs one thread's MMAs in issue order, so
      // the projection cannot overwrite phi'(a) before the contraction has read it.
      if (lane == 0) {
        const int w = warp - 1;
        const uint32_t tw = tbase + w * C::T_WG;
        const uint32_t dQ = tw + C::T_Q, dU = tw + C::T_U, dO = tw + C::T_O;
        const uint32_t id1 = idesc_f16(128, C::FB, false, false);
        const uint32_t id2 = idesc_f16(128, C::NROWS, false, false);
        const int ntw = (n - w + 1) / 2;  // my tiles
        const int nblk = ntw * nb;
        int a1 = 0, t1 = 0, j1 = 0;  // next projection: block a1 = t1 * nb + j1
        auto issue_mma1 = [&]() -> bool {
          if (j1 == 0 && !mbar_wait(bar(C::B_CVT + 2 * w + (t1 & 1)), (t1 >> 1) & 1, abort_flag, err)) return false;
          // No wait for MMA2(a1 - 2), which reads phi' from the same columns: this thread issued it
          // just before, and the tensor core executes one thread's MMAs in issue order.
          tc_fence_after();
          const uint32_t d = dU + (a1 & 1) * C::FB;
#pragma unroll
          for (int ks = 0; ks < C::D / 16; ++ks)
            mma_ts(d, dQ + 8 * ks, sdesc_sw128(sbase + C::S_W + (C::FB * j1) * 128 + 32 * ks, 16, 1024), id1,
                   ks > 0 ? 1u : 0u);
          mma_commit(bar(C::B_UF + 2 * w + (a1 & 1)));
          if (j1 == nb - 1) mma_commit(bar(C::B_QT + w));  // the Q operand may take my next tile
          ++a1;
          if (++j1 == nb) {
            j1 = 0;
            ++t1;
          }
          return true;
        };
        int rel = 0;  // images below rel released by me
        // releases image rel without having used it (after its predecessor's release completed,
        // so that the arrival counts towards the right phase)
        auto release_unused = [&]() {
          if (rel >= 1 && !mbar_wait(bar(C::B_SE), (rel - 1) & 1, abort_flag, err)) return false;
          mbar_arrive(bar(C::B_SE));
          ++rel;
          return true;
        };
        bool ok = true;
        for (int i = 0; i < 2 && a1 < nblk && ok; ++i) ok = issue_mma1();
        TileCursor cur;
        if (ntw > 0) cur.init(T0 + w, ntq, G, kvh0);
        // images before my first one are never mine: release them at once
        while (ok && ntw > 0 && rel < cur.img) ok = release_unused();
        for (int b = 0, j = 0, tc = 0; b < nblk && ok; ++b) {
          const int k = cur.img;
          if (!mbar_wait(bar(C::B_PHI + 2 * w + (b & 1)), (b >> 1) & 1, abort_flag, err)) break;
          if (j == 0) {
            // O is free once the previous tile has been read out; this tile's image must be in
            if (tc >= 1 && !mbar_wait(bar(C::B_OE + w), (tc - 1) & 1, abort_flag, err)) break;
            if (!wait_count_above(img_count, k, abort_flag, err)) break;
          }
          tc_fence_after();
          const uint32_t aP = dU + (b & 1) * C::FB;
#pragma unroll
          for (int ks = 0; ks < C::FB / 16; ++ks)  // O += phi' S', 16 features per step, two per column
            mma_ts(dO, aP + 8 * ks,
                   sdesc_sw128(sbase + C::S_SP + j * (C::NROWS * 128) + 32 * ks, 16, 1024), id2,
                   (j > 0 || ks > 0) ? 1u : 0u);
          mma_commit(bar(C::B_M2 + 2 * w + (b & 1)));
          if (j == nb - 1) {
            mma_commit(bar(C::B_OF + w));
            TileCursor nx = cur;  // my next tile
            nx.step(2, ntq, G);
            const int knext = tc + 1 < ntw ? nx.img : nimg;
            if (knext > k && k < nimg - 1) {  // done with image k: released when these MMAs complete
              mma_commit(bar(C::B_SE));
              rel = k + 1;
            }
            // images between this one and my next one are never mine: release them now, before
            // waiting for anything of my next tile (the image warp needs them to load my next image)
            while (ok && rel < min(knext, nimg - 1)) ok = release_unused();
            cur = nx;
            ++tc;
            j = 0;
          } else {
            ++j;
          }
          if (a1 < nblk) ok = issue_mma1();  // block b + 2, into the buffer MMA2(b) just read
        }
        while (ok && rel < nimg - 1) ok = release_unused();
        if (nblk >= 1) mbar_wait(bar(C::B_M2 + 2 * w + ((nblk - 1) & 1)), ((nblk - 1) >> 1) & 1, abort_flag, err, 200000000ull);
      }
    }
  } else if (warp < C::CVT0) {
    setmaxnreg_inc<C::R_EPI>();
    // ---------------- epilogue warpgroup w: tiles w, w + 2, ... ----------------
    const int eq = warp & 3;
    const int w = (warp - C::EPI0) >> 2;
    const int r = eq * 32 + lane;  // query row within the tile (TMEM lane)
    const uint32_t cU = w * C::T_WG + C::T_U, cO = w * C::T_WG + C::T_O;
    const float* ev = reinterpret_cast<const float*>(smem + C::S_SP + C::NROWS * 128 * nb);  // e_f, -inf past m
    const int ntw = (n - w + 1) / 2;
    TileCursor ec;
    if (ntw > 0) ec.init(T0 + w, ntq, G, kvh0);
    for (int tc = 0, b = 0; tc < ntw; ++tc, ec.step(2, ntq, G)) {
      wait_count_above(img_count, ec.img, abort_flag, err);                           // this tile's image is in
      mbar_wait(bar(C::B_CVT + 2 * w + (tc & 1)), (tc >> 1) & 1, abort_flag, err);  // its row scales are written
      const float up = upv[(w * 4 + (tc & 3)) * 128 + r];
      const float2 up2 = make_float2(up, up);
      float c = 0.f;
      for (int j = 0; j < nb; ++j, ++b) {
        mbar_wait(bar(C::B_UF + 2 * w + (b & 1)), (b >> 1) & 1, abort_flag, err);
        tc_fence_after();
        const uint32_t cb = cU + (b & 1) * C::FB;
        float v[C::FB];
        tmem_ld32(taddr(tbase, eq, cb), *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld32(taddr(tbase, eq, cb + 32), *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_wait_ld();
        const float4* e4p = reinterpret_cast<const float4*>(ev + C::FB * j);
        uint32_t ph[C::FB / 2];
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        // phi' = 2^(v - c) for the whole block, as fp16 pairs
        auto exponentiate = [&]() {
          const float2 nc2 = make_float2(-c, -c);
#pragma unroll
          for (int k2 = 0; k2 < C::FB / 2; ++k2) {
            const float2 bb = __fadd2_rn(make_float2(v[2 * k2], v[2 * k2 + 1]), nc2);
            ph[k2] = pack_f16x2(ex2(bb.x), ex2(bb.y));
          }
        };
        if constexpr (RELU) {
          // t = max(U, 0) 2^k 2^e_f and its maximum; phi' = t 2^-c
#pragma unroll
          for (int k4 = 0; k4 < C::FB / 4; ++k4) {
            const float4 s4 = e4p[k4];  // 2^e_f
            v[4 * k4 + 0] = fmaxf(v[4 * k4 + 0], 0.f) * (up * s4.x);
            v[4 * k4 + 1] = fmaxf(v[4 * k4 + 1], 0.f) * (up * s4.y);
            v[4 * k4 + 2] = fmaxf(v[4 * k4 + 2], 0.f) * (up * s4.z);
            v[4 * k4 + 3] = fmaxf(v[4 * k4 + 3], 0.f) * (up * s4.w);
            m4[k4 & 3] = fmax3(m4[k4 & 3], v[4 * k4 + 0], v[4 * k4 + 1]);
            m4[k4 & 3] = fmax3(m4[k4 & 3], v[4 * k4 + 2], v[4 * k4 + 3]);
          }
          const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
          // the integer c = E(mx) - 14 puts the block's largest phi' in [2^14, 2^15) (a row of zeros keeps c)
          const int cm = mx > 0.f ? ((__float_as_int(mx) >> 23) & 0xFF) - 127 - 14 : -1000;
          if (j == 0) {
            c = mx > 0.f ? static_cast<float>(max(-120, min(120, cm))) : 0.f;
          } else {
            const bool need = cm > static_cast<int>(c);
            if (__any_sync(0xffffffffu, need)) {  // cold: raise c for those rows, rescale the contractions so far
              mbar_wait(bar(C::B_M2 + 2 * w + ((b - 1) & 1)), ((b - 1) >> 1) & 1, abort_flag, err);
              tc_fence_after();
              const int cn = need ? min(120, cm) : static_cast<int>(c);
              scale_tmem_row(taddr(tbase, eq, cO), C::NROWS / 8,
                             __int_as_float((127 + max(-126, static_cast<int>(c) - cn)) << 23));
              c = static_cast<float>(cn);
            }
          }
          const float rc = __int_as_float((127 - static_cast<int>(c)) << 23);  // 2^-c
#pragma unroll
          for (int k2 = 0; k2 < C::FB / 2; ++k2) ph[k2] = pack_f16x2(v[2 * k2] * rc, v[2 * k2 + 1] * rc);
        } else
        // v = 2^k U + e (a feature past m has W' = 0 and e = -inf: v = -inf), and its maximum
        if (j == 0) {  // the row's first block: its exact maximum first, then the exponentials
#pragma unroll
          for (int k4 = 0; k4 < C::FB / 4; ++k4) {
            const float4 e4 = e4p[k4];
            const float2 v01 = __ffma2_rn(make_float2(v[4 * k4 + 0], v[4 * k4 + 1]), up2, make_float2(e4.x, e4.y));
            const float2 v23 = __ffma2_rn(make_float2(v[4 * k4 + 2], v[4 * k4 + 3]), up2, make_float2(e4.z, e4.w));
            v[4 * k4 + 0] = v01.x;
            v[4 * k4 + 1] = v01.y;
            v[4 * k4 + 2] = v23.x;
            v[4 * k4 + 3] = v23.y;
            m4[k4 & 3] = fmax3(m4[k4 & 3], v01.x, v01.y);
            m4[k4 & 3] = fmax3(m4[k4 & 3], v23.x, v23.y);
          }
          c = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
          exponentiate();
        } else {  // one pass with the row's stabiliser, the block's maximum alongside
          const float2 nc2 = make_float2(-c, -c);
#pragma unroll
          for (int k4 = 0; k4 < C::FB / 4; ++k4) {
            const float4 e4 = e4p[k4];
            const float2 v01 = __ffma2_rn(make_float2(v[4 * k4 + 0], v[4 * k4 + 1]), up2, make_float2(e4.x, e4.y));
            const float2 v23 = __ffma2_rn(make_float2(v[4 * k4 + 2], v[4 * k4 + 3]), up2, make_float2(e4.z, e4.w));
            v[4 * k4 + 0] = v01.x;
            v[4 * k4 + 1] = v01.y;
            v[4 * k4 + 2] = v23.x;
            v[4 * k4 + 3] = v23.y;
            m4[k4 & 3] = fmax3(m4[k4 & 3], v01.x, v01.y);
            m4[k4 & 3] = fmax3(m4[k4 & 3], v23.x, v23.y);
            const float2 b01 = __fadd2_rn(v01, nc2), b23 = __fadd2_rn(v23, nc2);
            ph[2 * k4] = pack_f16x2(ex2(b01.x), ex2(b01.y));
            ph[2 * k4 + 1] = pack_f16x2(ex2(b23.x), ex2(b23.y));
          }
          const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
          const bool need = mx > c + C::kRaise;
          if (__any_sync(0xffffffffu, need)) {  // cold: this block would overflow fp16 for some row
            // raise c for those rows: the contractions so far (outputs and normaliser) are rescaled
            // once the previous block's contraction has completed, then the block is redone
            mbar_wait(bar(C::B_M2 + 2 * w + ((b - 1) & 1)), ((b - 1) >> 1) & 1, abort_flag, err);
            tc_fence_after();
            scale_tmem_row(taddr(tbase, eq, cO), C::NROWS / 8, need ? ex2(c - mx) : 1.f);
            if (need) c = mx;
            exponentiate();
          }
        }
        // phi' as fp16 pairs over the first 32 columns of this block's U buffer
        tmem_st16(taddr(tbase, eq, cb), *reinterpret_cast<uint32_t(*)[16]>(&ph[0]));
        tmem_st16(taddr(tbase, eq, cb + 16), *reinterpret_cast<uint32_t(*)[16]>(&ph[16]));
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::B_PHI + 2 * w + (b & 1)));
      }
    }
  } else {
    setmaxnreg_dec<C::R_CVT>();
    // ---------------- converter / output warpgroup ----------------
    const int q = warp & 3;
    const int r = q * 32 + lane;  // row within a tile (TMEM lane)
    // Q tile t (local order; warpgroup t % 2) into its warpgroup's tensor-memory operand as fp16 x
    // 2^-k, k = 0 unless the row's largest |q| reaches 2^15, when it brings it into [2^14, 2^15);
    // 2^k goes to shared memory for the epilogue.  Thread r starts at chunk r % 8 so that the
    // eight threads of a shared-memory wavefront hit different banks.
    auto convert = [&](int t) {
      const int w = t & 1, tcw = t >> 1, s = t % NQS;
      mbar_wait(bar(C::B_QF + s), (t / NQS) & 1, abort_flag, err);
      if (tcw >= 1) mbar_wait(bar(C::B_QT + w), (tcw - 1) & 1, abort_flag, err);  // the operand is free
      const unsigned char* qrow = smem + C::S_Q + s * C::QTILE + r * 128;
      uint4 v[8];
      uint32_t emax = 0;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        v[c] = *reinterpret_cast<const uint4*>(qrow + 16 * (c ^ (r & 7)));
        emax = __vmaxu2(emax, v[c].x & 0x7FFF7FFFu);
        emax = __vmaxu2(emax, v[c].y & 0x7FFF7FFFu);
        emax = __vmaxu2(emax, v[c].z & 0x7FFF7FFFu);
        emax = __vmaxu2(emax, v[c].w & 0x7FFF7FFFu);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_QE + s));  // this warp has read its rows of the stage
      // the biased bf16 exponent of the row's largest |q|
      const int ebits = static_cast<int>(max(emax & 0xFFFFu, emax >> 16) >> 7);
      // the ReLU map is scale-free per row, so its small rows are scaled up as well (a row of zeros
      // keeps k = -100 and stays zero)
      const int k = min(100, max(RELU ? -100 : 0, ebits - 141));
      const bool plain = __all_sync(0xffffffffu, k == 0);
      const float down = __int_as_float((127 - k) << 23);
      uint32_t o[32];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t wv[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float lo = __uint_as_float(wv[e] << 16), hi = __uint_as_float(wv[e] & 0xFFFF0000u);
          if (!plain) {
            lo *= down;
            hi *= down;
          }
          o[4 * c + e] = pack_f16x2(lo, hi);
        }
      }
      tmem_st32(taddr(tbase, q, w * C::T_WG + C::T_Q), o);
      upv[(w * 4 + (tcw & 3)) * 128 + r] = __int_as_float((127 + k) << 23);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_CVT + 2 * w + (tcw & 1)));  // this warp's 32 rows are in
    };
    unsigned char* slot = smem + C::S_STG + q * 4096;
    // tile t's output: O / normaliser -> bf16 -> this warp's staging slot -> TMA store
    auto output = [&](int t, int qt, int bh) {
      const int w = t & 1, tcw = t >> 1;
      mbar_wait(bar(C::B_OF + w), tcw & 1, abort_flag, err);
      tc_fence_after();
      const uint32_t cO = w * C::T_WG + C::T_O;
      uint32_t o[32], dn[8];
      tmem_ld8(taddr(tbase, q, cO + C::D), dn);  // the normaliser
      tmem_ld32(taddr(tbase, q, cO), o);
      tmem_wait_ld();
      const float inv = 1.f / __uint_as_float(dn[0]);
      if (lane == 0) bulk_wait_read<0>();  // this warp's previous store has read the slot
      __syncwarp();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (h == 1) {
          tmem_ld32(taddr(tbase, q, cO + 32), o);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(C::B_OE + w));  // O may take the warpgroup's next tile
        }
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w4[e] = pack_bf16x2(__uint_as_float(o[8 * c4 + 2 * e]) * inv, __uint_as_float(o[8 * c4 + 2 * e + 1]) * inv);
          const int c8 = 4 * h + c4;
          *reinterpret_cast<uint4*>(slot + lane * 128 + ((c8 ^ (lane & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_3d(&tmO, smem_u32(slot), 0, qt * 128 + 32 * q, bh);
        bulk_commit();
      }
    };
    for (int t = 0; t < min(n, 2); ++t) convert(t);
    TileCursor oc;
    if (n > 0) oc.init(T0, ntq, G, kvh0);
    for (int t = 0; t < n; ++t, oc.step(1, ntq, G)) {
      if (t + 2 < n) convert(t + 2);
      output(t, oc.qt, oc.bh);
    }
    if (lane == 0) bulk_wait<0>();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, 512);
}
