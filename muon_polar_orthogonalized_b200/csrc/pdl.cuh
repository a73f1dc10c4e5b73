// pdl.cuh -- programmatic dependent launch for every kernel of the library.
//
// Each kernel is launched with programmatic stream serialization allowed, so
// the GPU may schedule it while the kernel before it in the stream is still
// finishing: its launch and its prologue (barrier setup, TMEM allocation)
// overlap the previous kernel's tail.  In exchange each kernel calls
// pdl_wait() before its first global-memory access: griddepcontrol.wait
// returns once every grid it depends on has completed and its writes are
// visible (at once when there is no such grid, e.g. after a memset or a
// library kernel launched without the attribute).  pdl_launch_dependents()
// lets the next kernel be scheduled; it runs nothing of it early, since that
// kernel waits in turn.  The elementwise kernels call it at their start
// (their blocks fill an SM's threads, so the next kernel's blocks only take
// the SMs they leave); the GEMMs call it after their last tile, since blocks
// of a next kernel placed beside a running GEMM CTA would take issue slots
// from it.
#pragma once
#include <cuda_runtime.h>

#include <utility>

namespace muon {

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// kernel<<<grid, block, smem, s>>>(args...) with the attribute set.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
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
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace muon
