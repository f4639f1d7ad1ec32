// Overlapped launches of consecutive kernels on one stream (programmatic dependent launch).
//
// Within one library call the state reduction and the query pass go out with the
// programmatic stream-serialisation attribute: each may be scheduled as soon as every CTA of
// the kernel before it (the call's own key pass or reduction) has started
// (griddep_launch_dependents) or exited, so its set-up (barrier initialisation,
// tensor-memory allocation, the W' fill, the first TMA loads of its own inputs) runs while
// that kernel's last CTAs finish.  Each kernel executes griddep_wait() before it reads
// anything that an earlier kernel of the sequence writes and before it writes anything that
// an earlier kernel reads; griddep_wait returns once the kernels it depends on have
// completed and their writes are visible, and at once for an ordinary launch.  The hardware
// schedules a dependent kernel only after every CTA of the earlier one is resident, so a
// waiting CTA never holds an SM that the earlier kernel still needs.
//
// The first kernel of a call reads its inputs (Q, K, V, W) before any wait, and the kernel
// before it on the stream is the caller's, which may let its dependents start before its own
// writes are done.  So that kernel is an ordinary launch unless the caller opts in
// (favor_set_launch_overlap); the later kernels of the call read their inputs early only
// after the first one has started, that is, after all of the caller's earlier work completed.
#pragma once

#include <cuda_runtime.h>

#include <utility>

namespace favor {

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// overlap = false gives an ordinary launch (the kernel starts once all earlier work on the
// stream has completed; its griddepcontrol instructions then do nothing).
template <typename... KArgs, typename... Args>
cudaError_t launch_overlapped(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              bool overlap, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = overlap ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace favor
