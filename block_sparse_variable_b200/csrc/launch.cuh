// launch.cuh -- programmatic dependent launch between the library's kernels.
//
// Every kernel of a call is launched with programmatic stream serialization:
// its CTAs may be placed on the SMs while the kernel before it in the stream
// is still finishing, and wait there (griddep_wait, the first thing each
// kernel does) until that kernel has completed and its writes are visible.
// Each kernel then lets the next one be placed (griddep_launch_next), which
// takes effect once all of its own CTAs have started, so a waiting CTA never
// holds resources that a CTA of the kernel it waits for still needs.  What
// this removes is the launch gap between consecutive small kernels.
#pragma once

#include <cuda_runtime.h>

#include <utility>

namespace bsa {

// wait for the preceding grid of the stream (a no-op for a plain launch)
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }

// allow the next grid of the stream to be scheduled
__device__ __forceinline__ void griddep_launch_next() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_dep(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace bsa
