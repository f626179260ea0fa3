// pdl.cuh -- programmatic dependent launch between two kernels of one call.
//
// The second kernel is launched with the programmatic-stream-serialisation
// attribute (launch_after_pdl), so that its CTAs may start while the first
// kernel's last CTAs are still running: once every CTA of the first kernel
// has executed pdl_launch_dependents (or exited), the second grid is
// scheduled as SMs free up.  Whatever in the second kernel reads memory the
// first kernel writes must come after pdl_wait, which returns once the first
// grid has completed and its writes are visible.
#pragma once
#include <cuda_runtime.h>

namespace eio {

__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launch kernel(args...) on stream s as a programmatic dependent of the
// kernel launched before it on s.
template <typename... KArgs, typename... Args>
cudaError_t launch_after_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             Args&&... args) {
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
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

}  // namespace eio
