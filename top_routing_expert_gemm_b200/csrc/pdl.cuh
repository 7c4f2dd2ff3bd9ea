// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may be scheduled before its predecessor in the stream has
// finished, and waits inside for it.  Used to chain the kernels of a
// decode-sized layer step, where launch latency is a visible share of the time.
//
// Rules every kernel here follows: a kernel that can be launched this way
// calls grid_dependency_wait() before it reads anything its predecessor
// writes, and calls grid_launch_dependents() (which lets its own successor be
// scheduled) only after that wait, so a kernel's set-up may still read what
// the launches before its predecessor wrote.  Both are no-ops for a launch
// without the attribute.
#pragma once

#include <cuda_runtime.h>

#include <utility>

namespace moe {

__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launch `kernel` on `stream`, programmatically dependent on the previous
// launch when `chained`.
template <typename... KArgs, typename... Args>
cudaError_t launch_maybe_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                 bool chained, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = chained ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace moe
