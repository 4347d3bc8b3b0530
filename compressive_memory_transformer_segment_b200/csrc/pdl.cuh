// Programmatic dependent launch (sm_90+): a kernel of the forward's chain may
// be launched while its predecessor in the stream is still running; it does
// its prologue (barrier setup, TMEM allocation, constant shared-memory
// panels), then waits until the predecessor grid has completed and its
// memory is visible before it touches global memory at all (inputs the
// caller wrote, workspace a previous call still reads).  Each kernel also
// lets its own successor launch as soon as all of its CTAs have started.
#pragma once

#include <cuda_runtime.h>

#include <utility>

namespace infini {

// Blocks until every prerequisite grid has completed and flushed its memory
// (returns at once when the kernel was launched without the attribute).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Allows the next kernel in the stream to be launched (it still waits in
// pdl_wait for this grid to complete).
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launch, with programmatic stream serialization when `pdl` is set.  Only
// kernels that call pdl_wait() before their first global memory access may
// be launched so.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace infini
