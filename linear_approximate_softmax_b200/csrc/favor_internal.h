// Internal declarations shared by the C-ABI layer and the kernels.
#pragma once

#include <cmath>
#include <cstddef>
#include <cstdint>

#include "favor.h"

struct CUstream_st;
typedef struct CUstream_st* cudaStream_t;

namespace favor {

// Records `msg` as the calling thread's last error and returns `code`.
int set_error(int code, const char* msg);
int set_errorf(int code, const char* fmt, ...);

int make_features(uint64_t seed, int m, int d, int orthogonal, float* W_out);

constexpr double kLog2e = 1.4426950408889634074;
constexpr int kTileTokens = 128;   // key chunks are whole multiples of this
constexpr int kStabBlock = 1;      // partial stabilisers are kept per feature

// How the key pass splits each kv head's L tokens into P chunks.
struct Plan {
  int B, H, Hkv, L, d, m;
  int P;            // chunks per kv head
  int chunk;        // tokens per chunk (multiple of kTileTokens, last one ragged)
  int nsb;          // stabilisers per partial: ceil(m / kStabBlock) = m
  // byte offsets inside the partials buffer
  size_t part_S_off, part_c_off, part_bytes;
  // byte offsets inside the state buffer
  size_t st_S_off, st_c_off, st_op_off, st_bytes;
  // The state re-packed as the fp16 B operand of the query pass's second MMA.
  // Per kv head: op_atoms blocks of 64 features, each op_rows rows (output column n; for
  // d = 64 rows d .. d + 15 follow: the normaliser column, then zeros) of 128 B, K-major
  // with the 128-byte swizzle (16-byte chunk c of row n
  // at c ^ (n % 8)); then e[op_tail] and the normaliser column s[op_tail], fp32, with
  // op_tail = m rounded up to 128.  Feature f's values are 2^-x_f S[f][n] relative to
  // its own largest chunk stabiliser c_f, with x_f chosen so that the largest lands in
  // [2^14, 2^15); e[f] = x_f + c_f - c*, and e[f] = -inf for f >= m, so that the query
  // pass needs no masking of the features past m.
  int op_rows, op_atoms, op_tail;
  size_t op_bytes;
  float wscale;     // d^-1/4 * log2(e): W is multiplied by this on the device
  float nscale;     // d^-1/2 * log2(e) / 2: |k|^2 is multiplied by this
};

// Fills `p` for a validated shape on the current device.  Returns FAVOR_OK or an error.
int make_plan(int B, int H, int Hkv, int L, int d, int m, Plan* p);

// Re-splits the key pass of `p` into at most max_P chunks per kv head and
// recomputes the partials layout (the state layout does not depend on it).
void plan_limit_chunks(Plan* p, int max_P);
// Re-splits the key chunks into P of them (as near as whole 128-token tiles allow).
void plan_set_chunks(Plan* p, int P);

// The three steps of the path, each dispatched to its kernel on `st`.  overlap: launch the
// kernel so that it may start while the kernel before it on `st` finishes (it waits before it
// touches that kernel's data, but reads its own inputs at once).  Within one call the library
// sets it for the kernels after the first; for the first kernel of a call it follows
// launch_overlap_enabled().
int run_key_pass(int dtype, const void* K, const void* V, const float* W, void* partials, const Plan& p,
                 cudaStream_t st, bool overlap);
int run_reduce(const void* partials, void* state, const Plan& p, cudaStream_t st, bool overlap);
int run_query_pass(int dtype, const void* Q, const float* W, const void* state, void* out, const Plan& p,
                   cudaStream_t st, bool overlap);
// favor_set_launch_overlap's setting (default off).
bool launch_overlap_enabled();

// ---- CUDA-core kernels (fp32 arithmetic; fp32 or bf16 storage) -------------
int simt_key_pass(int dtype, const void* K, const void* V, const float* W, void* partials,
                  const Plan& p, void* stream);
int simt_state_reduce(const void* partials, void* state, const Plan& p, void* stream, bool overlap);
int simt_query_pass(int dtype, const void* Q, const float* W, const void* state, void* out,
                    const Plan& p, void* stream);
// The same key and query passes with the feature map f = ReLU (no stabilisers); the
// reduction is shared.
int simt_key_pass_relu(int dtype, const void* K, const void* V, const float* W, void* partials, const Plan& p,
                       void* stream);
int simt_query_pass_relu(int dtype, const void* Q, const float* W, const void* state, void* out, const Plan& p,
                         void* stream);
// Linformer projected attention on the same machinery: the projections E K, F V of each kv
// head written as key-pass partials of 2 * heads heads (plan pk: 2B batches), reduced by
// simt_state_reduce, then the query pass with the exp map over the k projected keys (plan pq).
int simt_linformer_proj(int dtype, const void* K, const void* V, const float* E, const float* F, void* partials,
                        const Plan& pk, int heads, void* stream);
int simt_linformer_query(int dtype, const void* Q, const void* state, void* out, const Plan& pq, const Plan& pk,
                         void* stream);

// ---- tensor-core kernels (sm_100a, bf16 storage) ------------------------------
bool sm100_key_supported(const Plan& p);
// Features per CTA of the tensor-core key pass: 256 for d = 64 with m > 128 (each of its two
// epilogue warpgroups takes 128 features of every key tile), else 128.
inline int key_features_per_cta(int d, int m) { return d == 64 && m > 128 ? 256 : 128; }
bool sm100_query_supported(const Plan& p);
int sm100_key_pass(const void* K, const void* V, const float* W, void* partials, const Plan& p, cudaStream_t st,
                   bool overlap);
// The tensor-core key and query passes with the feature map f = ReLU (bf16, d = 64; the query
// pass for 64 < m <= 512).
int sm100_key_pass_relu(const void* K, const void* V, const float* W, void* partials, const Plan& p, cudaStream_t st);
int sm100_query_pass_relu(const void* Q, const float* W, const void* state, void* out, const Plan& p, cudaStream_t st);
// Linformer's projections E K and F V on the tensor cores (d = 64): E and F split into bf16 hi + lo
// in `split` (linformer_split_bytes), then the partial states of the plan's 2 heads kv heads.
size_t linformer_split_bytes(int kp, int L);
int sm100_linformer_proj(const void* K, const void* V, const float* E, const float* F, void* split, void* partials,
                         const Plan& pk, int heads, cudaStream_t st);
// Linformer's projected query pass on the tensor cores (bf16, d = 64, 64 < k <= 512): the query
// pass of each kv head with its projected keys as W and its projected values as the state.
int sm100_linformer_query(const void* Q, const void* state, void* out, const Plan& pq, const Plan& pk, cudaStream_t st);
// W's scale for the ReLU map: d^-1/4 (the exponential map's carries log2(e) as well).
inline float relu_wscale(int d) { return static_cast<float>(1.0 / std::sqrt(std::sqrt(static_cast<double>(d)))); }
int sm100_query_pass(const void* Q, const float* W, const void* state, void* out, const Plan& p, cudaStream_t st,
                     bool overlap);
// Reads and clears the device error word (bit 0: a bounded wait gave up).
int sm100_read_and_clear_error(unsigned int* word);

}  // namespace favor
