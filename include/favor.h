/*
 * favor.h — C ABI of the B200 (sm_100a) FAVOR+ attention library.
 *
 * FAVOR+ ("Rethinking Attention with Performers", Abstract and section
 * 제안 방법 / proposed method) estimates softmax attention with positive
 * orthogonal random features in time and memory linear in the sequence length:
 *
 *   x'      = d^(-1/4) x                     (queries and keys)
 *   phi(x') = exp(W x' - |x'|^2/2) / sqrt(m) (W: m x d random features)
 *   out     = phi(Q') (phi(K')^T [V | 1]) / (last column)
 *
 * and the L x L attention matrix is never formed.  Query head h reads key/value
 * head h / (H / Hkv): the multi-query layout of "Fast Transformer Decoding:
 * One Write-Head is All You Need" (提出的方法 / proposed method) when Hkv = 1.
 *
 * Conventions shared by every entry point:
 *  - Return 0 (FAVOR_OK) on success, a negative FAVOR_ERR_* code on failure;
 *    favor_last_error() then holds a message (thread-local).  Nothing throws
 *    across the ABI and no argument error launches any GPU work.
 *  - Tensors are dense, contiguous, row-major:
 *      Q, out [B, H, L, d];  K, V [B, Hkv, L, d];  W [m, d] fp32.
 *  - Device pointers must be 16-byte aligned (FAVOR_ERR_INVALID otherwise).
 *  - The caller owns every buffer it passes; the library keeps no pointer to
 *    any of them after a call returns.
 *  - GPU entry points are asynchronous on `stream` (0 = legacy default
 *    stream) and never synchronise it; CUDA launch errors are reported as
 *    FAVOR_ERR_CUDA.
 *  - Within one call, the state reduction and the tensor-core query pass are
 *    launched with programmatic dependent launch: each may start while the
 *    call's kernel before it finishes, and waits (griddepcontrol.wait) before
 *    it reads or overwrites memory that kernel uses.  The first kernel of a
 *    call is an ordinary launch (it starts once all earlier work on `stream`
 *    has completed) unless favor_set_launch_overlap(1) was called.  Work the
 *    caller adds to `stream` afterwards is ordered after the call as usual; a
 *    kernel the caller launches with programmatic stream serialisation must
 *    wait the same way before it reads the call's outputs.
 *  - Supported shapes: d in {64, 128}; m a multiple of 16 with 16 <= m <= 512;
 *    B, H, Hkv, L >= 1; H % Hkv == 0; B * H <= 65535.  Anything else is
 *    FAVOR_ERR_UNSUPPORTED.
 */
#ifndef FAVOR_B200_H
#define FAVOR_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* favor_stream_t; /* the same type as cudaStream_t */

#if defined(__GNUC__)
#define FAVOR_API __attribute__((visibility("default")))
#else
#define FAVOR_API
#endif

#define FAVOR_OK 0
#define FAVOR_ERR_INVALID (-1)     /* null or misaligned pointer, bad size or flag   */
#define FAVOR_ERR_UNSUPPORTED (-2) /* shape outside the supported set (see above)     */
#define FAVOR_ERR_CUDA (-3)        /* a CUDA runtime call or launch failed            */
#define FAVOR_ERR_NOMEM (-4)       /* a host or device allocation failed              */
#define FAVOR_ERR_TIMEOUT (-5)     /* a GPU kernel gave up waiting (see favor_device_check) */

/* Element type of Q, K, V and out. */
#define FAVOR_BF16 0
#define FAVOR_F32 1

/*
 * favor_set_launch_overlap — how the first kernel of every later call starts
 * (process-wide; returns the previous setting, 0 or 1).
 *
 * 0 (the default): an ordinary launch, after all earlier work on the stream.
 * 1: a programmatic dependent launch, like the later kernels of a call: it may
 * start as soon as the kernel before it on the stream lets its dependents start
 * (griddepcontrol.launch_dependents) or exits, and it reads its inputs (Q, K, V,
 * W, or a stage call's partial state or state) at once, before that kernel's
 * writes are guaranteed to be visible.  The library's own kernels let their
 * dependents start at entry.  So with 1, NO INPUT OF A CALL MAY BE WRITTEN BY THE
 * KERNEL JUST BEFORE IT ON THE STREAM when that kernel is one of this library's
 * (for example, the out of one call fed as Q, K or V of the next, as in stacked
 * layers) or any other kernel that lets its dependents start early; chained calls
 * like these need 0, or an event or any ordinary kernel launch between them.
 * Kernels that do not use programmatic dependent launch never let dependents
 * start early, so after them 1 is safe.  A call's set-up then overlaps the end of
 * the kernel before it (for back-to-back calls on independent inputs, the
 * previous query pass).
 */
FAVOR_API int favor_set_launch_overlap(int enable);

/* Message for the last non-zero return on the calling thread ("" if none). */
FAVOR_API const char* favor_last_error(void);

/* Library version, e.g. 100 for 0.1.0. */
FAVOR_API int favor_version(void);

/*
 * favor_device_check — synchronise `stream`, then read and clear the library's
 * device error word.  The tensor-core kernels bound every wait inside their
 * pipelines; a CTA that gives up (after 2 s) stops, frees its tensor memory and
 * sets the word, and its outputs are then undefined.  Returns FAVOR_OK,
 * FAVOR_ERR_TIMEOUT if any kernel gave up since the last check, or
 * FAVOR_ERR_CUDA.  The word is per device and shared by all streams.
 */
FAVOR_API int favor_device_check(favor_stream_t stream);

/*
 * favor_make_features — the random-feature matrix W (host only, no GPU).
 *
 * "Rethinking Attention with Performers", Abstract / 제안 방법: positive
 * orthogonal random features.  orthogonal != 0: ceil(m/d) independent d x d
 * blocks of standard normals, rows orthonormalised first to last by
 * Gram-Schmidt in fp64 (each projection applied twice); the first m rows of
 * the stacked blocks are kept and row r is scaled to the length |h_r| of an
 * independent h_r ~ N(0, I_d), so every row is marginally N(0, I_d).
 * orthogonal == 0: the first m rows of the same normal stream, unchanged.
 *
 * Random numbers: Philox4x64-10 (Salmon et al., SC'11) with key (seed, 0);
 * the n-th normal of stream t comes from counter (n/4, t, 0, 0) through
 * Box-Muller on u = ((x >> 12) + 1/2) 2^-52.  Stream 0 feeds the blocks,
 * stream 1 the norm vectors.  The same (seed, m, d, orthogonal) always gives
 * the same W, on any machine, up to the last bit of the fp64 libm.
 *
 * W_out: host, caller-owned, m*d floats, row-major [m, d], written as the fp64
 * result rounded to fp32.  W is passed to the attention calls UNSCALED.
 * Errors: FAVOR_ERR_INVALID (null W_out, m < 1, d < 1),
 * FAVOR_ERR_NOMEM (scratch allocation failed).  Any m, d >= 1 is accepted.
 */
FAVOR_API int favor_make_features(uint64_t seed, int m, int d, int orthogonal, float* W_out);

/*
 * favor_attention — bf16 FAVOR+ attention, bidirectional (device pointers).
 *
 * Q [B,H,L,d], K and V [B,Hkv,L,d] bf16; W [m,d] fp32 (unscaled, as
 * favor_make_features writes it); out [B,H,L,d] bf16.  Accumulation is fp32.
 * The path: key pass (phi(K') and per-chunk partial states phi(K')^T [V|1],
 * each with its own max stabiliser), a fixed-order reduction that rescales the
 * partials to one stabiliser (bitwise deterministic), then the query pass
 * (phi(Q') with a per-row stabiliser, the product with the state, and the
 * division by the last column).  The scratch memory it needs (partials and
 * the state) is allocated and freed stream-ordered on `stream`
 * (cudaMallocAsync / cudaFreeAsync); FAVOR_ERR_CUDA if that fails.
 */
FAVOR_API int favor_attention(const void* Q, const void* K, const void* V, const float* W, void* out,
                    int B, int H, int Hkv, int L, int d, int m, favor_stream_t stream);

/* favor_attention_f32 — the same with fp32 Q, K, V and out (fp32 arithmetic
 * throughout, no tensor-core rounding). */
FAVOR_API int favor_attention_f32(const float* Q, const float* K, const float* V, const float* W, float* out,
                        int B, int H, int Hkv, int L, int d, int m, favor_stream_t stream);

/*
 * favor_attention_relu — generalised kernelizable attention with f = ReLU.
 *
 * "Rethinking Attention with Performers" (Abstract; 연구 질문 / research
 * questions, RQ5): the same linear-time scheme approximates attention with
 * kernels other than softmax.  The pages name no f; this is the plainest one:
 * phi(x) = max(W x', 0) / sqrt(m), x' = d^-1/4 x, with the same W, and
 * out = phi(Q')(phi(K')^T V) / (phi(Q')(phi(K')^T 1)).  The scalings cancel in
 * the ratio (ReLU is positively homogeneous) and no stabiliser is needed.
 * dtype FAVOR_BF16 or FAVOR_F32 for Q, K, V and out; arguments, layouts,
 * shapes, scratch and errors as favor_attention.  It runs on the CUDA cores in
 * fp32 (key pass per chunk, the fixed-order reduction, query pass).  A query
 * whose features meet no key's (denominator 0) gets inf or nan, as the
 * division gives.
 */
FAVOR_API int favor_attention_relu(int dtype, const void* Q, const void* K, const void* V, const float* W,
                         void* out, int B, int H, int Hkv, int L, int d, int m, favor_stream_t stream);

/*
 * favor_linformer — Linformer projected attention (a second workload on the
 * same machinery).
 *
 * Linformer notes page, section "4 Model": keys and values are projected along
 * the sequence by E and F (k x L), and attention runs over the k projected
 * rows: out = softmax(Q (E K)^T / sqrt(d)) (F V), per head.  One E and one F
 * serve every head (the shared-projection option); query head h uses kv head
 * h / (H / Hkv)'s projected rows.  E, F: device fp32 [kp, L] row-major (the
 * caller's; random N(0, 1/L) entries stand in for trained ones).  dtype FAVOR_BF16 or
 * FAVOR_F32 for Q, K, V and out; their layouts and the shape limits are those
 * of favor_attention with m = kp (a multiple of 16 in [16, 512]) and, in
 * addition, 2 * B * H <= 65535.  It runs on the CUDA cores in fp32: a
 * projection kernel that sums each chunk of tokens into partial products, the
 * fixed-order reduction, and the query pass with the exponential map over the
 * kp projected keys (the softmax: a per-row maximum, exp, the weighted sum of
 * F V and the division by the sum of the weights).  Scratch is allocated and
 * freed stream-ordered on `stream`; errors as favor_attention.
 */
FAVOR_API int favor_linformer(int dtype, const void* Q, const void* K, const void* V, const float* E,
                    const float* F, void* out, int B, int H, int Hkv, int L, int d, int kp,
                    favor_stream_t stream);

/*
 * favor_attention_host — end-to-end call on HOST buffers.
 *
 * Q, K, V, out are host pointers (pinned memory gives asynchronous copies;
 * pageable memory works, slower); W is a host [m,d] fp32 array.  dtype is
 * FAVOR_BF16 or FAVOR_F32 for Q, K, V and out.  The call splits the B*Hkv kv
 * heads into at most 8 pieces of consecutive kv heads (each with its H/Hkv
 * query heads, one contiguous range of every tensor), copies each piece in on
 * an internal host-to-device stream, computes it on `stream` as a problem of
 * its own (B = 1; the result equals favor_attention(_f32) on those heads bit
 * for bit) and copies it out on an internal device-to-host stream, so that both
 * copy directions and the compute overlap.  It synchronises `stream` before
 * returning.  Device buffers (two pieces' tensors, W, one piece's scratch) are
 * allocated and freed stream-ordered on `stream` inside the call; the two copy
 * streams are created on first use per device and kept for the process.
 */
FAVOR_API int favor_attention_host(int dtype, const void* Q, const void* K, const void* V, const float* W,
                         void* out, int B, int H, int Hkv, int L, int d, int m,
                         favor_stream_t stream);

/* ---------------------------------------------------------------------------
 * Stage-level calls.  favor_attention == favor_key_pass + favor_state_reduce +
 * favor_query_pass on one stream, with the caller providing the scratch.
 * ------------------------------------------------------------------------- */

/* Bytes of key-pass partials for this shape on the current device (the chunk
 * count depends on the device's SM count).  0 for unsupported shapes. */
FAVOR_API size_t favor_partials_bytes(int B, int Hkv, int L, int d, int m);

/*
 * Bytes of the reduced state for B*Hkv kv heads.  Layout (fp32 unless noted):
 *   S    [B*Hkv][m][d+1]   phi(K')^T [V | 1] scaled by 2^(-c) (c per kv head)
 *   c    [B*Hkv]           the key stabiliser, in log2 units
 *   then an internal region (the state re-packed as tensor-core operands),
 *   written by favor_state_reduce and read by favor_query_pass.
 * 0 for unsupported shapes.
 */
FAVOR_API size_t favor_state_bytes(int B, int Hkv, int d, int m);

/* favor_key_pass — phi(K') and the partial states of every key chunk.
 * dtype: FAVOR_BF16 or FAVOR_F32 (element type of K and V).  partials: device,
 * caller-owned, favor_partials_bytes(...) bytes, fully overwritten. */
FAVOR_API int favor_key_pass(int dtype, const void* K, const void* V, const float* W, void* partials,
                   int B, int Hkv, int L, int d, int m, favor_stream_t stream);

/* favor_state_reduce — rescale the partials of each kv head to the largest
 * chunk stabiliser and sum them in chunk order (bitwise deterministic).
 * state: device, caller-owned, favor_state_bytes(...) bytes, fully overwritten. */
FAVOR_API int favor_state_reduce(const void* partials, void* state, int B, int Hkv, int L, int d, int m,
                       favor_stream_t stream);

/* favor_query_pass — out = phi(Q') S[:, :d] / phi(Q') S[:, d] for every query
 * head, reading the state of kv head h / (H/Hkv).  dtype as for the key pass
 * (element type of Q and out). */
FAVOR_API int favor_query_pass(int dtype, const void* Q, const float* W, const void* state, void* out,
                     int B, int H, int Hkv, int L, int d, int m, favor_stream_t stream);

/*
 * favor_attention_noalloc — favor_attention for callers that cannot allocate.
 *
 * The pages have no counterpart to this call; it serves the library's users.
 * favor_attention allocates its scratch on every call.  A caller whose device
 * memory is owned and budgeted by its own allocator, or whose serving loop
 * cannot afford an allocator call, uses this entry point instead: it computes
 * the same result and allocates nothing, using a 16 MiB array in device
 * global memory that is part of the library (every GPU that loads the
 * library's kernels holds it until the process exits).
 *
 * dtype: FAVOR_BF16 or FAVOR_F32 for Q, K, V and out; other arguments as for
 * favor_attention (device pointers, caller-owned, 16-byte aligned).
 * The first call on each device looks up the array's device address (with
 * that device current); make that first call before any stream capture.
 * To fit, the key pass may be split into fewer chunks than favor_attention
 * uses, so results can differ from it in the last bits.  Shapes whose state
 * alone does not fit return FAVOR_ERR_UNSUPPORTED with the sizes in
 * favor_last_error().  Every call shares the one array and overwrites all of
 * the scratch it uses, so nothing has to be cleared between calls, but calls
 * that overlap on the GPU (on different streams, or from different threads)
 * race on it: serialise them.  The looked-up address belongs to the device's
 * primary context of the process: after cudaDeviceReset (or any teardown of that
 * context) this entry point must not be called again in the same process.
 */
FAVOR_API int favor_attention_noalloc(int dtype, const void* Q, const void* K, const void* V, const float* W,
                                      void* out, int B, int H, int Hkv, int L, int d, int m,
                                      favor_stream_t stream);

/* ---------------------------------------------------------------------------
 * Incremental decoding against a cached state.
 *
 * "Fast Transformer Decoding: One Write-Head is All You Need" (研究动机与目标 /
 * motivation, 提出的方法 / proposed method): one token at a time, every step
 * reads the whole cache of each key/value head, and H query heads may share one
 * key/value head.  With FAVOR+ the cache of a kv head is its state: a fixed
 * m x (d + 1) matrix plus one stabiliser per feature, whatever the number of
 * tokens seen ("Rethinking Attention with Performers", Abstract: linear space).
 * ------------------------------------------------------------------------- */

/* Bytes of a decode state for B*Hkv kv heads.  Layout per kv head (fp32):
 *   S [m][d+1]   sum over the tokens seen of 2^(a_t,f - c_f) [v_t | 1], with
 *                a_t,f = d^-1/4 log2(e) W_f . k_t - d^-1/2 log2(e) |k_t|^2 / 2
 *   c [m]        the largest a_t,f seen for each feature (-inf before the first token)
 * so that exp(...) of the method = 2^(a) and S relative to 2^c.
 * 0 for unsupported shapes (see favor_decode_step). */
FAVOR_API size_t favor_decode_state_bytes(int B, int Hkv, int d, int m);

/* favor_decode_init — the empty state (S = 0, c = -inf) of B*Hkv kv heads, on `stream`.
 * state: device, caller-owned, favor_decode_state_bytes(...) bytes, 16-byte aligned. */
FAVOR_API int favor_decode_init(void* state, int B, int Hkv, int d, int m, favor_stream_t stream);

/*
 * favor_decode_step — one decoding step for every sequence of the batch.
 *
 * Appends key/value k, v [B, Hkv, d] (one token per kv head) to the state, then
 * answers the queries q [B, H, d] (query head h reads kv head h / (H / Hkv))
 * against the updated state: out [B, H, d] = FAVOR+ attention of each query over
 * every token appended so far, including this one.  dtype: FAVOR_BF16 or
 * FAVOR_F32 for q, k, v and out; W [m, d] fp32 unscaled; state as above, updated
 * in place (the stabiliser update is exact: c_f is the running maximum and S is
 * rescaled whenever it rises).  All pointers device, caller-owned, 16-byte
 * aligned.  Shapes: d in {64, 128}; m a multiple of 16 in [16, 512]; H % Hkv == 0
 * with at most 64 query heads per kv head.  Each kv head is one cluster of 8 CTAs
 * on the CUDA cores (fp32 arithmetic throughout).  Asynchronous on `stream`;
 * calls on one state must be ordered (each reads the state the previous one wrote).
 */
FAVOR_API int favor_decode_step(int dtype, const void* q, const void* k, const void* v, const float* W,
                                void* state, void* out, int B, int H, int Hkv, int d, int m,
                                favor_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FAVOR_B200_H */
