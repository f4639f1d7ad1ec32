// C ABI of the FAVOR+ library: argument checks, planning, scratch and dispatch.
// Every exported function is declared and documented in include/favor.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <atomic>
#include <mutex>
#include <string>
#include <vector>

#include "favor_internal.h"

namespace favor {

namespace {
thread_local std::string g_last_error;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shape(int B, int H, int Hkv, int L, int d, int m) {
  if (B < 1 || H < 1 || Hkv < 1 || L < 1)
    return set_errorf(FAVOR_ERR_UNSUPPORTED, "B, H, Hkv and L must be >= 1 (got %d, %d, %d, %d)", B, H, Hkv, L);
  if (H % Hkv != 0) return set_errorf(FAVOR_ERR_UNSUPPORTED, "H (%d) must be a multiple of Hkv (%d)", H, Hkv);
  if (d != 64 && d != 128) return set_errorf(FAVOR_ERR_UNSUPPORTED, "d must be 64 or 128 (got %d)", d);
  if (m < 16 || m > 512 || m % 16 != 0)
    return set_errorf(FAVOR_ERR_UNSUPPORTED, "m must be a multiple of 16 in [16, 512] (got %d)", m);
  // the kernels index (batch, head) pairs with a grid dimension of at most 65535
  if (static_cast<long>(B) * H > 65535)
    return set_errorf(FAVOR_ERR_UNSUPPORTED, "B * H must be at most 65535 (got %ld)", static_cast<long>(B) * H);
  const double elems = static_cast<double>(B) * H * L * d;
  if (elems > 4.0e12) return set_error(FAVOR_ERR_UNSUPPORTED, "tensor too large");
  return FAVOR_OK;
}

int check_dtype(int dtype) {
  if (dtype != FAVOR_BF16 && dtype != FAVOR_F32)
    return set_errorf(FAVOR_ERR_INVALID, "dtype must be FAVOR_BF16 (0) or FAVOR_F32 (1), got %d", dtype);
  return FAVOR_OK;
}

int check_ptrs(const char* what, std::initializer_list<const void*> ptrs) {
  for (const void* p : ptrs) {
    if (!p) return set_errorf(FAVOR_ERR_INVALID, "%s: null pointer argument", what);
    if (!aligned16(p)) return set_errorf(FAVOR_ERR_INVALID, "%s: pointer %p is not 16-byte aligned", what, p);
  }
  return FAVOR_OK;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int device_sm_count(int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "no usable CUDA device: %s", cudaGetErrorString(e));
  return FAVOR_OK;
}

#define FAVOR_TRY(expr)            \
  do {                             \
    int _rc = (expr);              \
    if (_rc != FAVOR_OK) return _rc; \
  } while (0)

#define FAVOR_CUDA_TRY(expr, what)                                                      \
  do {                                                                                  \
    cudaError_t _e = (expr);                                                            \
    if (_e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "%s: %s", what, cudaGetErrorString(_e)); \
  } while (0)

}  // namespace

int set_error(int code, const char* msg) {
  g_last_error = msg ? msg : "";
  return code;
}

int set_errorf(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int make_plan(int B, int H, int Hkv, int L, int d, int m, Plan* p) {
  FAVOR_TRY(check_shape(B, H, Hkv, L, d, m));
  int sms = 0;
  FAVOR_TRY(device_sm_count(&sms));
  p->B = B; p->H = H; p->Hkv = Hkv; p->L = L; p->d = d; p->m = m;
  const int heads = B * Hkv;
  const int tiles = (L + kTileTokens - 1) / kTileTokens;
  // Key chunks: the tensor-core key pass runs one CTA per SM for each (kv head,
  // feature group, chunk).  Pick the chunk count that minimises the
  // makespan in waves of CTAs, counting half a tile of start-up per wave, plus the
  // partial state the chunks write and the reduction reads back (about 4 MB in the
  // time a CTA spends on one key tile).
  const int nfeat = key_features_per_cta(d, m);
  const long units = static_cast<long>(heads) * ((m + nfeat - 1) / nfeat);
  constexpr double kPartBytesPerTile = 4.0e6;
  double best = 1e300;
  int best_ct = tiles;
  for (int P = 1; P <= tiles; ++P) {
    const int ct = (tiles + P - 1) / P;
    const long Pe = (tiles + ct - 1) / ct;
    if (Pe != P) continue;
    const long waves = (units * Pe + sms - 1) / sms;
    const double part_bytes = static_cast<double>(heads) * Pe * m * (d + 1) * sizeof(float);
    const double cost = static_cast<double>(waves) * (ct + 0.5) + part_bytes / kPartBytesPerTile;
    if (cost < best - 1e-9) { best = cost; best_ct = ct; }
  }
  p->chunk = best_ct * kTileTokens;
  p->P = (tiles + best_ct - 1) / best_ct;
  p->nsb = (m + kStabBlock - 1) / kStabBlock;
  const size_t D1 = static_cast<size_t>(d) + 1;
  p->part_S_off = 0;
  p->part_c_off = round_up(sizeof(float) * heads * p->P * m * D1, 256);
  p->part_bytes = p->part_c_off + round_up(sizeof(float) * heads * p->P * p->nsb, 256);
  p->st_S_off = 0;
  p->st_c_off = round_up(sizeof(float) * heads * m * D1, 256);
  p->st_op_off = p->st_c_off + round_up(sizeof(float) * heads, 256);
  // the query pass's state operand: d rows of fp16, and for d = 64 the normaliser as row d and 15
  // rows of zeros (the tensor-core query pass reads them as 16 more output columns)
  p->op_rows = d == 64 ? d + 16 : d;
  p->op_atoms = (m + 63) / 64;
  p->op_tail = (m + 127) / 128 * 128;
  // fp16 rows (64 features per 128-byte row), then one fp32 exponent per feature, then the
  // fp32 normaliser column with the same per-feature scaling
  p->op_bytes = static_cast<size_t>(p->op_rows) * 128 * p->op_atoms + 8 * static_cast<size_t>(p->op_tail);
  p->st_bytes = p->st_op_off + round_up(p->op_bytes * heads, 256);
  p->wscale = static_cast<float>(std::pow(static_cast<double>(d), -0.25) * kLog2e);
  p->nscale = static_cast<float>(std::pow(static_cast<double>(d), -0.5) * kLog2e * 0.5);
  return FAVOR_OK;
}

void plan_limit_chunks(Plan* p, int max_P) {
  if (max_P < 1) max_P = 1;
  if (p->P <= max_P) return;
  plan_set_chunks(p, max_P);
}

void plan_set_chunks(Plan* p, int P) {
  const int heads = p->B * p->Hkv;
  const int tiles = (p->L + kTileTokens - 1) / kTileTokens;
  const int chunk_tiles = (tiles + std::max(1, std::min(P, tiles)) - 1) / std::max(1, std::min(P, tiles));
  p->chunk = chunk_tiles * kTileTokens;
  p->P = (tiles + chunk_tiles - 1) / chunk_tiles;
  const size_t D1 = static_cast<size_t>(p->d) + 1;
  p->part_c_off = round_up(sizeof(float) * heads * p->P * p->m * D1, 256);
  p->part_bytes = p->part_c_off + round_up(sizeof(float) * heads * p->P * p->nsb, 256);
}

int run_key_pass(int dtype, const void* K, const void* V, const float* W, void* partials, const Plan& p,
                 cudaStream_t st, bool overlap) {
  if (dtype == FAVOR_BF16 && sm100_key_supported(p)) return sm100_key_pass(K, V, W, partials, p, st, overlap);
  return simt_key_pass(dtype, K, V, W, partials, p, st);  // an ordinary launch
}

int run_reduce(const void* partials, void* state, const Plan& p, cudaStream_t st, bool overlap) {
  return simt_state_reduce(partials, state, p, st, overlap);
}

int run_query_pass(int dtype, const void* Q, const float* W, const void* state, void* out, const Plan& p,
                   cudaStream_t st, bool overlap) {
  if (dtype == FAVOR_BF16 && sm100_query_supported(p)) return sm100_query_pass(Q, W, state, out, p, st, overlap);
  return simt_query_pass(dtype, Q, W, state, out, p, st);  // an ordinary launch
}

namespace {
std::atomic<int> g_launch_overlap{0};
}  // namespace

bool launch_overlap_enabled() { return g_launch_overlap.load(std::memory_order_relaxed) != 0; }

namespace {

// Stream-ordered scratch is returned to the device's default pool after each
// call; by default the pool unmaps it at the next synchronisation, so the
// next call maps it again.  Keep it mapped (once per device, this process only).
void keep_pool_mapped() {
  static bool done[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 || done[dev]) return;
  cudaMemPool_t pool;
  if (cudaDeviceGetDefaultMemPool(&pool, dev) == cudaSuccess) {
    uint64_t threshold = UINT64_MAX;
    cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &threshold);
  }
  done[dev] = true;
}

// The host-buffer call's copy streams on each device (host to device, device to host),
// created on first use and kept for the process, so that the two copy directions run on
// their own copy engines beside the compute on the caller's stream.
int copy_streams(cudaStream_t* in, cudaStream_t* out) {
  static std::mutex mu;
  static cudaStream_t streams[64][2] = {};
  int dev = 0;
  FAVOR_CUDA_TRY(cudaGetDevice(&dev), "favor_attention_host device");
  if (dev < 0 || dev >= 64) return set_error(FAVOR_ERR_UNSUPPORTED, "favor_attention_host: device index above 63");
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < 2; ++i)
    if (!streams[dev][i])
      FAVOR_CUDA_TRY(cudaStreamCreateWithFlags(&streams[dev][i], cudaStreamNonBlocking), "favor_attention_host streams");
  *in = streams[dev][0];
  *out = streams[dev][1];
  return FAVOR_OK;
}

int attention_impl(int dtype, const void* Q, const void* K, const void* V, const float* W, void* out, int B,
                   int H, int Hkv, int L, int d, int m, cudaStream_t st) {
  FAVOR_TRY(check_dtype(dtype));
  FAVOR_TRY(check_ptrs("favor_attention", {Q, K, V, W, out}));
  Plan p;
  FAVOR_TRY(make_plan(B, H, Hkv, L, d, m, &p));
  keep_pool_mapped();
  void* ws = nullptr;
  const size_t st_off = round_up(p.part_bytes, 256);
  FAVOR_CUDA_TRY(cudaMallocAsync(&ws, st_off + p.st_bytes, st), "favor_attention scratch allocation");
  char* base = static_cast<char*>(ws);
  int rc = run_key_pass(dtype, K, V, W, base, p, st, launch_overlap_enabled());
  if (rc == FAVOR_OK) rc = run_reduce(base, base + st_off, p, st, true);
  if (rc == FAVOR_OK) rc = run_query_pass(dtype, Q, W, base + st_off, out, p, st, true);
  cudaError_t fe = cudaFreeAsync(ws, st);
  if (rc != FAVOR_OK) return rc;
  FAVOR_CUDA_TRY(fe, "favor_attention scratch release");
  return FAVOR_OK;
}

// phi = ReLU(W x'): the same plan and scratch, the CUDA-core key and query passes with the
// ReLU map, the shared reduction.
int relu_attention_impl(int dtype, const void* Q, const void* K, const void* V, const float* W, void* out, int B,
                        int H, int Hkv, int L, int d, int m, cudaStream_t st) {
  FAVOR_TRY(check_dtype(dtype));
  FAVOR_TRY(check_ptrs("favor_attention_relu", {Q, K, V, W, out}));
  Plan p;
  FAVOR_TRY(make_plan(B, H, Hkv, L, d, m, &p));
  keep_pool_mapped();
  void* ws = nullptr;
  const size_t st_off = round_up(p.part_bytes, 256);
  FAVOR_CUDA_TRY(cudaMallocAsync(&ws, st_off + p.st_bytes, st), "favor_attention_relu scratch allocation");
  char* base = static_cast<char*>(ws);
  // bf16 with d = 64: the tensor-core key pass with the map swapped; otherwise the CUDA-core one
  int rc = dtype == FAVOR_BF16 && d == 64 ? sm100_key_pass_relu(K, V, W, base, p, st)
                                          : simt_key_pass_relu(dtype, K, V, W, base, p, st);
  if (rc == FAVOR_OK) rc = run_reduce(base, base + st_off, p, st, false);
  if (rc == FAVOR_OK)
    rc = dtype == FAVOR_BF16 && d == 64 && m > 64 && m <= 512
             ? sm100_query_pass_relu(Q, W, base + st_off, out, p, st)
             : simt_query_pass_relu(dtype, Q, W, base + st_off, out, p, st);
  cudaError_t fe = cudaFreeAsync(ws, st);
  if (rc != FAVOR_OK) return rc;
  FAVOR_CUDA_TRY(fe, "favor_attention_relu scratch release");
  return FAVOR_OK;
}

// Linformer projected attention: projection kernel -> reduction -> projected query pass.
int linformer_impl(int dtype, const void* Q, const void* K, const void* V, const float* E, const float* F,
                   void* out, int B, int H, int Hkv, int L, int d, int kp, cudaStream_t st) {
  FAVOR_TRY(check_dtype(dtype));
  FAVOR_TRY(check_ptrs("favor_linformer", {Q, K, V, E, F, out}));
  if (2L * B * H > 65535) return set_error(FAVOR_ERR_UNSUPPORTED, "favor_linformer: 2 * B * H must be at most 65535");
  Plan pq, pk;
  FAVOR_TRY(make_plan(B, H, Hkv, L, d, kp, &pq));
  FAVOR_TRY(make_plan(2 * B, H, Hkv, L, d, kp, &pk));  // the projected keys ride as B more batches
  // bf16 with d = 64: the projections on the tensor cores, in enough key chunks for about two
  // waves of CTAs (128 projected rows x chunk x product x 4 kv heads each)
  const bool tc = dtype == FAVOR_BF16 && d == 64;
  if (tc) {
    int sms = 0;
    FAVOR_TRY(device_sm_count(&sms));
    const long per_chunk = static_cast<long>((kp + 127) / 128) * 2 * ((B * Hkv + 3) / 4);
    plan_set_chunks(&pk, static_cast<int>(std::max(1L, (2L * sms + per_chunk - 1) / per_chunk)));
  }
  keep_pool_mapped();
  void* ws = nullptr;
  const size_t st_off = round_up(pk.part_bytes, 256);
  const size_t split_off = st_off + round_up(pk.st_bytes, 256);
  const size_t ws_bytes = split_off + (tc ? linformer_split_bytes(kp, L) : 0);
  FAVOR_CUDA_TRY(cudaMallocAsync(&ws, ws_bytes, st), "favor_linformer scratch allocation");
  char* base = static_cast<char*>(ws);
  int rc = tc ? sm100_linformer_proj(K, V, E, F, base + split_off, base, pk, B * Hkv, st)
              : simt_linformer_proj(dtype, K, V, E, F, base, pk, B * Hkv, st);
  if (rc == FAVOR_OK) rc = run_reduce(base, base + st_off, pk, st, false);
  if (rc == FAVOR_OK)
    rc = dtype == FAVOR_BF16 && d == 64 && kp > 64 && kp <= 512 ? sm100_linformer_query(Q, base + st_off, out, pq, pk, st)
                                                               : simt_linformer_query(dtype, Q, base + st_off, out, pq, pk, st);
  cudaError_t fe = cudaFreeAsync(ws, st);
  if (rc != FAVOR_OK) return rc;
  FAVOR_CUDA_TRY(fe, "favor_linformer scratch release");
  return FAVOR_OK;
}

}  // namespace
}  // namespace favor

using namespace favor;

extern "C" {

const char* favor_last_error(void) { return g_last_error.c_str(); }

int favor_version(void) { return 100; }

int favor_set_launch_overlap(int enable) {
  return g_launch_overlap.exchange(enable ? 1 : 0, std::memory_order_relaxed);
}

int favor_make_features(uint64_t seed, int m, int d, int orthogonal, float* W_out) {
  return make_features(seed, m, d, orthogonal, W_out);
}

int favor_attention(const void* Q, const void* K, const void* V, const float* W, void* out, int B, int H,
                    int Hkv, int L, int d, int m, favor_stream_t stream) {
  return attention_impl(FAVOR_BF16, Q, K, V, W, out, B, H, Hkv, L, d, m, reinterpret_cast<cudaStream_t>(stream));
}

int favor_attention_f32(const float* Q, const float* K, const float* V, const float* W, float* out, int B, int H,
                        int Hkv, int L, int d, int m, favor_stream_t stream) {
  return attention_impl(FAVOR_F32, Q, K, V, W, out, B, H, Hkv, L, d, m, reinterpret_cast<cudaStream_t>(stream));
}

int favor_attention_relu(int dtype, const void* Q, const void* K, const void* V, const float* W, void* out, int B,
                         int H, int Hkv, int L, int d, int m, favor_stream_t stream) {
  return relu_attention_impl(dtype, Q, K, V, W, out, B, H, Hkv, L, d, m, reinterpret_cast<cudaStream_t>(stream));
}

int favor_linformer(int dtype, const void* Q, const void* K, const void* V, const float* E, const float* F, void* out,
                    int B, int H, int Hkv, int L, int d, int kp, favor_stream_t stream) {
  return linformer_impl(dtype, Q, K, V, E, F, out, B, H, Hkv, L, d, kp, reinterpret_cast<cudaStream_t>(stream));
}

int favor_attention_host(int dtype, const void* Q, const void* K, const void* V, const float* W, void* out, int B,
                         int H, int Hkv, int L, int d, int m, favor_stream_t stream) {
  FAVOR_TRY(check_dtype(dtype));
  if (!Q || !K || !V || !W || !out) return set_error(FAVOR_ERR_INVALID, "favor_attention_host: null pointer argument");
  FAVOR_TRY(check_shape(B, H, Hkv, L, d, m));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaStream_t s_in = nullptr, s_out = nullptr;
  FAVOR_TRY(copy_streams(&s_in, &s_out));
  // Pieces of consecutive kv heads (each with its G query heads): kv head t = b * Hkv + j owns
  // query heads t * G .. t * G + G - 1 in the [B, H] order, so a piece is one contiguous range of
  // Q, K, V and out and is computed as a problem of its own (B = 1).  Piece i goes in on s_in,
  // is computed on the caller's stream and goes out on s_out, double-buffered on the device, so
  // the copies of neighbouring pieces overlap each other (both directions) and the compute.
  const int G = H / Hkv, KH = B * Hkv;
  const int NP = KH < 8 ? KH : 8;
  const int nmax = (KH + NP - 1) / NP;
  const size_t es = dtype == FAVOR_F32 ? 4 : 2;
  const size_t row = static_cast<size_t>(L) * d * es;  // one head of one tensor
  const size_t bkv = round_up(nmax * row, 256), bq = round_up(nmax * G * row, 256);
  const size_t bw = round_up(sizeof(float) * m * d, 256);
  auto piece = [&](int i, int* t0, int* n) {
    *t0 = static_cast<int>(static_cast<long>(KH) * i / NP);
    *n = static_cast<int>(static_cast<long>(KH) * (i + 1) / NP) - *t0;
  };
  size_t part_max = 0, st_max = 0;  // one scratch for every piece's partials and state
  for (int i = 0; i < NP; ++i) {
    int t0, n;
    piece(i, &t0, &n);
    Plan pp;
    FAVOR_TRY(make_plan(1, n * G, n, L, d, m, &pp));
    part_max = pp.part_bytes > part_max ? pp.part_bytes : part_max;
    st_max = pp.st_bytes > st_max ? pp.st_bytes : st_max;
  }
  const size_t st_off = round_up(part_max, 256);
  const size_t scratch = st_off + round_up(st_max, 256);
  const size_t slot = 2 * bkv + 2 * bq;  // K, V, Q, out of one piece
  keep_pool_mapped();
  void* buf = nullptr;
  FAVOR_CUDA_TRY(cudaMallocAsync(&buf, bw + scratch + 2 * slot, st), "favor_attention_host device allocation");
  char* dW = static_cast<char*>(buf);
  char* dS = dW + bw;
  std::vector<cudaEvent_t> ev(3 * NP + 1, nullptr);  // ready, then per piece: in, computed, out
  cudaError_t e = cudaSuccess;
  for (auto& x : ev)
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&x, cudaEventDisableTiming);
  auto ev_in = [&](int i) { return ev[1 + 3 * i]; };
  auto ev_comp = [&](int i) { return ev[2 + 3 * i]; };
  auto ev_out = [&](int i) { return ev[3 + 3 * i]; };
  int rc = FAVOR_OK;
  if (e == cudaSuccess) e = cudaEventRecord(ev[0], st);  // the allocation (and all earlier work on st)
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s_in, ev[0], 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, ev[0], 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dW, W, sizeof(float) * m * d, cudaMemcpyHostToDevice, s_in);
  if (e != cudaSuccess) rc = set_errorf(FAVOR_ERR_CUDA, "favor_attention_host set-up: %s", cudaGetErrorString(e));
  for (int i = 0; i < NP && rc == FAVOR_OK; ++i) {
    int t0, n;
    piece(i, &t0, &n);
    char* sK = dS + scratch + (i & 1) * slot;
    char* sV = sK + bkv;
    char* sQ = sV + bkv;
    char* sO = sQ + bq;
    const size_t nkv = n * row, nq = static_cast<size_t>(n) * G * row;
    if (i >= 2) e = cudaStreamWaitEvent(s_in, ev_comp(i - 2), 0);  // piece i - 2 has read this slot
    if (e == cudaSuccess) e = cudaMemcpyAsync(sK, static_cast<const char*>(K) + t0 * row, nkv, cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess) e = cudaMemcpyAsync(sV, static_cast<const char*>(V) + t0 * row, nkv, cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(sQ, static_cast<const char*>(Q) + static_cast<size_t>(t0) * G * row, nq, cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess) e = cudaEventRecord(ev_in(i), s_in);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ev_in(i), 0);
    if (e == cudaSuccess && i >= 2) e = cudaStreamWaitEvent(st, ev_out(i - 2), 0);  // this slot's output has left
    if (e != cudaSuccess) {
      rc = set_errorf(FAVOR_ERR_CUDA, "favor_attention_host copy in: %s", cudaGetErrorString(e));
      break;
    }
    Plan pp;
    rc = make_plan(1, n * G, n, L, d, m, &pp);
    const float* w = reinterpret_cast<const float*>(dW);
    // the key pass follows an event wait on the stream: an ordinary launch
    if (rc == FAVOR_OK) rc = run_key_pass(dtype, sK, sV, w, dS, pp, st, false);
    if (rc == FAVOR_OK) rc = run_reduce(dS, dS + st_off, pp, st, true);
    if (rc == FAVOR_OK) rc = run_query_pass(dtype, sQ, w, dS + st_off, sO, pp, st, true);
    if (rc != FAVOR_OK) break;
    e = cudaEventRecord(ev_comp(i), st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, ev_comp(i), 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(static_cast<char*>(out) + static_cast<size_t>(t0) * G * row, sO, nq, cudaMemcpyDeviceToHost, s_out);
    if (e == cudaSuccess) e = cudaEventRecord(ev_out(i), s_out);
    if (e != cudaSuccess) {
      rc = set_errorf(FAVOR_ERR_CUDA, "favor_attention_host copy out: %s", cudaGetErrorString(e));
      break;
    }
  }
  // join both copy streams into the caller's stream (also after an error), then release
  cudaEvent_t jin = nullptr, jout = nullptr;
  cudaError_t je = cudaEventCreateWithFlags(&jin, cudaEventDisableTiming);
  if (je == cudaSuccess) je = cudaEventCreateWithFlags(&jout, cudaEventDisableTiming);
  if (je == cudaSuccess) je = cudaEventRecord(jin, s_in);
  if (je == cudaSuccess) je = cudaEventRecord(jout, s_out);
  if (je == cudaSuccess) je = cudaStreamWaitEvent(st, jin, 0);
  if (je == cudaSuccess) je = cudaStreamWaitEvent(st, jout, 0);
  if (je != cudaSuccess) {  // cannot order the release after the copies: wait for them here
    cudaStreamSynchronize(s_in);
    cudaStreamSynchronize(s_out);
  }
  cudaError_t fe = cudaFreeAsync(buf, st);
  cudaError_t se = cudaStreamSynchronize(st);
  for (auto& x : ev)
    if (x) cudaEventDestroy(x);
  if (jin) cudaEventDestroy(jin);
  if (jout) cudaEventDestroy(jout);
  if (rc != FAVOR_OK) return rc;
  if (je != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "favor_attention_host join: %s", cudaGetErrorString(je));
  if (fe != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "favor_attention_host release: %s", cudaGetErrorString(fe));
  if (se != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "favor_attention_host: %s", cudaGetErrorString(se));
  return FAVOR_OK;
}

int favor_device_check(favor_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "favor_device_check: %s", cudaGetErrorString(e));
  unsigned int word = 0;
  FAVOR_TRY(sm100_read_and_clear_error(&word));
  if (word) return set_errorf(FAVOR_ERR_TIMEOUT, "a tensor-core kernel gave up waiting (error word 0x%x)", word);
  return FAVOR_OK;
}

size_t favor_partials_bytes(int B, int Hkv, int L, int d, int m) {
  Plan p;
  if (make_plan(B, Hkv, Hkv, L, d, m, &p) != FAVOR_OK) return 0;
  return p.part_bytes;
}

size_t favor_state_bytes(int B, int Hkv, int d, int m) {
  Plan p;
  if (make_plan(B, Hkv, Hkv, 1, d, m, &p) != FAVOR_OK) return 0;
  return p.st_bytes;
}

int favor_key_pass(int dtype, const void* K, const void* V, const float* W, void* partials, int B, int Hkv, int L,
                   int d, int m, favor_stream_t stream) {
  FAVOR_TRY(check_dtype(dtype));
  FAVOR_TRY(check_ptrs("favor_key_pass", {K, V, W, partials}));
  Plan p;
  FAVOR_TRY(make_plan(B, Hkv, Hkv, L, d, m, &p));
  return run_key_pass(dtype, K, V, W, partials, p, reinterpret_cast<cudaStream_t>(stream), launch_overlap_enabled());
}

int favor_state_reduce(const void* partials, void* state, int B, int Hkv, int L, int d, int m,
                       favor_stream_t stream) {
  FAVOR_TRY(check_ptrs("favor_state_reduce", {partials, state}));
  Plan p;
  FAVOR_TRY(make_plan(B, Hkv, Hkv, L, d, m, &p));
  return run_reduce(partials, state, p, reinterpret_cast<cudaStream_t>(stream), launch_overlap_enabled());
}

int favor_query_pass(int dtype, const void* Q, const float* W, const void* state, void* out, int B, int H, int Hkv,
                     int L, int d, int m, favor_stream_t stream) {
  FAVOR_TRY(check_dtype(dtype));
  FAVOR_TRY(check_ptrs("favor_query_pass", {Q, W, state, out}));
  Plan p;
  FAVOR_TRY(make_plan(B, H, Hkv, L, d, m, &p));
  return run_query_pass(dtype, Q, W, state, out, p, reinterpret_cast<cudaStream_t>(stream),
                        launch_overlap_enabled());
}

}  // extern "C"
