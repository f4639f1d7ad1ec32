// favor_attention_noalloc: the FAVOR+ path with its scratch in a static device array.
//
// favor_attention takes its scratch (key-pass partials and the reduced state)
// from the stream-ordered allocator on every call.  Some callers cannot allow
// that: a framework that owns all device memory through its own caching
// allocator and budgets it up front, or a latency-critical serving loop where
// an allocator call (which may map new memory and synchronise) is not
// acceptable.  This entry point gives them the same computation with no
// allocation at all: the scratch lives in one file-scope __device__ array of
// kStaticScratchBytes, which every GPU that loads this library's kernels keeps
// until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "favor_internal.h"

namespace favor {
namespace {

// 16 MiB: the partials and the state of the five benchmark workloads fit after
// the key pass is re-split into fewer chunks when needed.
constexpr size_t kStaticScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices];  // device address of g_static_scratch per device, set up on first use

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// The device address of g_static_scratch on the current device.  In host code
// the array's name only stands in for the symbol, so its address has to be
// asked of the runtime once per device, with that device current.
int static_scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_errorf(FAVOR_ERR_CUDA, "favor_attention_noalloc: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return set_errorf(FAVOR_ERR_UNSUPPORTED, "favor_attention_noalloc: device %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || !p)
      return set_errorf(FAVOR_ERR_CUDA, "favor_attention_noalloc: cudaGetSymbolAddress failed: %s",
                        cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return FAVOR_OK;
}

}  // namespace
}  // namespace favor

using namespace favor;

extern "C" int favor_attention_noalloc(int dtype, const void* Q, const void* K, const void* V, const float* W,
                                       void* out, int B, int H, int Hkv, int L, int d, int m,
                                       favor_stream_t stream) {
  if (dtype != FAVOR_BF16 && dtype != FAVOR_F32)
    return set_errorf(FAVOR_ERR_INVALID, "favor_attention_noalloc: dtype must be 0 or 1, got %d", dtype);
  for (const void* ptr : {Q, K, V, static_cast<const void*>(W), static_cast<const void*>(out)})
    if (!ptr || (reinterpret_cast<uintptr_t>(ptr) & 15u))
      return set_error(FAVOR_ERR_INVALID, "favor_attention_noalloc: null or not 16-byte aligned pointer");
  Plan p;
  int rc = make_plan(B, H, Hkv, L, d, m, &p);
  if (rc != FAVOR_OK) return rc;
  // Fewer key chunks mean smaller partials; the state does not shrink.
  const size_t per_chunk = round256(p.part_bytes) / static_cast<size_t>(p.P) + 1;
  const size_t st_room = round256(p.st_bytes);
  if (st_room < kStaticScratchBytes) {
    const size_t room = kStaticScratchBytes - st_room;
    plan_limit_chunks(&p, static_cast<int>(room / per_chunk));
  }
  // the estimate above ignores the 256-byte rounding of each array: step down until it fits
  while (round256(p.part_bytes) + p.st_bytes > kStaticScratchBytes && p.P > 1) plan_limit_chunks(&p, p.P - 1);
  const size_t st_off = round256(p.part_bytes);
  if (st_off + p.st_bytes > kStaticScratchBytes)
    return set_errorf(FAVOR_ERR_UNSUPPORTED,
                      "favor_attention_noalloc: this shape needs %zu bytes of scratch; the static scratch holds %zu",
                      st_off + p.st_bytes, kStaticScratchBytes);
  void* scratch = nullptr;
  rc = static_scratch_address(&scratch);
  if (rc != FAVOR_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(scratch);
  rc = run_key_pass(dtype, K, V, W, base, p, st, launch_overlap_enabled());
  if (rc == FAVOR_OK) rc = run_reduce(base, base + st_off, p, st, true);
  if (rc == FAVOR_OK) rc = run_query_pass(dtype, Q, W, base + st_off, out, p, st, true);
  return rc;
}
