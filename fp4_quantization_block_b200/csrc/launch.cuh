// launch.cuh -- programmatic dependent launch for the library's kernels.
//
// Every kernel of the hot path is launched with programmatic stream
// serialization: it may be scheduled while the kernel before it in the
// stream is still finishing (its tail CTAs), run its prologue (barrier
// initialisation, tensor-memory allocation, tensor-map prefetch) on the SMs
// that have become free, and only then wait for the previous kernel with
// griddepcontrol.wait, before its first access to global memory.  Each
// kernel signals griddepcontrol.launch_dependents early, so the next one
// can be scheduled in the same way.  The wait returns only when the
// previous grid has completed and its memory operations are visible, so a
// kernel that follows any other work (ours or not) sees all of it; without
// the launch attribute the wait returns at once.
#pragma once

#include <cuda_runtime.h>

#include <utility>

namespace fa4 {

// Block until the previous grid in the stream has completed (every thread
// that touches global memory executes it first).
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Let the next grid in the stream be scheduled before this one completes.
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// The launch attribute that allows the overlap above.
inline cudaLaunchAttribute pdl_attribute() {
  cudaLaunchAttribute a;
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
  return a;
}

// kern<<<grid, block, smem, st>>>(args...) with the attribute.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace fa4
