// infini_attn_forward_noalloc: the layer forward for callers that cannot
// allocate GPU memory at call time.
//
// Who needs it.  Some callers may not call cudaMalloc / cudaMallocAsync (or an
// allocator that ends in them) while they run: code that executes inside a
// region where allocation is forbidden or would deadlock (a custom allocator's
// own callback, a real-time or interrupt-like loop that must not block on the
// driver's allocator, an embedding that owns all device memory through a
// fixed arena and does not expose it).  Such a caller still owns and passes its
// inputs and outputs, but it cannot hand this library a workspace.
//
// How.  The scratch the forward needs (the memory every segment reads, for
// all segments) lives in one file-scope device array of fixed size,
// kNoAllocScratchBytes.  Host code cannot use the array's name as a device
// address, so every call looks the address up with cudaGetSymbolAddress
// (with the caller's device current) and runs the regular forward with that
// address as its workspace.  The lookup is repeated on every call rather
// than cached: after cudaDeviceReset the module is loaded again, possibly at
// another address, and a cached pointer would be stale.  Nothing here
// allocates.
//
// First call per device.  CUDA loads a library's GPU code lazily by default
// (CUDA_MODULE_LOADING=LAZY): the first call on a device loads the modules
// this call uses, which commits device memory for their code and for the
// 64 MiB array.  A caller that must never allocate makes one warm-up call
// outside its no-allocation region (or runs with CUDA_MODULE_LOADING=EAGER);
// later calls of the same shape commit nothing.
#include <cuda_runtime.h>
#include <stdint.h>

#include "infini_attn.h"

namespace {

// 64 MiB: enough for the tiny, 200M-, 300M- and 8B-shaped workloads; a
// 1M-token stream needs about 1.7 GiB and is rejected.
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device.
cudaError_t scratch_address(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  *out = p;
  return cudaSuccess;
}

}  // namespace

extern "C" {

size_t infini_attn_noalloc_scratch_limit(void) { return kNoAllocScratchBytes; }

int infini_attn_forward_noalloc(const void* q, const void* k, const void* v, const float* beta,
                                const float* M_in, const float* z_in, int seg_len, int rule,
                                const infini_dims_t* dims, void* out, float* M_out, float* z_out,
                                void* stream) {
  const size_t need = infini_attn_workspace_bytes(dims, seg_len, rule);
  if (need == 0) {
    infini_plan_t plan;
    const int rc = infini_attn_plan(dims, seg_len, rule, &plan);
    return rc != INFINI_OK ? rc : INFINI_ERR_ARG;
  }
  if (need > kNoAllocScratchBytes) return INFINI_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return INFINI_ERR_CUDA;
  // Every byte of scratch the kernels read is written earlier in the same
  // call, so nothing has to be cleared between calls.
  return infini_attn_forward(q, k, v, beta, M_in, z_in, seg_len, rule, dims, out, M_out, z_out,
                             scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
