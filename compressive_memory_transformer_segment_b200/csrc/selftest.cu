// Self-checks: the device approximations the tensor-core attention kernel
// uses in place of library functions (the FMA-pipe 2^x, exp2_poly2, both of
// its lanes; the hardware 2^x, ex2.approx; the bf16 packing of
// probabilities), and the failure path of the kernels' bounded waits.
#include <cuda_runtime.h>

#include "infini_attn.h"
#include "kernels.h"
#include "tc_common.cuh"

namespace {

__global__ void selftest_kernel(const float* __restrict__ x, float* __restrict__ y_poly,
                                float* __restrict__ y_mufu, unsigned int* __restrict__ bf16_bits,
                                int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float v = x[i];
  const float2 p2 = infini::tc::exp2_poly2(make_float2(v, v));
  y_poly[i] = (i & 1) ? p2.y : p2.x;
  y_mufu[i] = infini::tc::ex2_approx(v);
  const float a = fabsf(v);
  bf16_bits[i] = infini::tc::pack_bf16x2(a, a) & 0xFFFFu;
}

// One warp waits on an mbarrier that nothing arrives at, with the kernels'
// bounded wait: it gives up after the time limit, sets the timeout bit of the
// status word and returns.
__global__ void selftest_timeout_kernel(unsigned int* __restrict__ status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    infini::tc::mbar_init(&bar, 1);
    abort_flag = 0;
    infini::tc::fence_mbar_init();
  }
  __syncthreads();
  const bool ok = __all_sync(0xffffffffu, infini::tc::mbar_wait(&bar, 0, &abort_flag, status));
  (void)ok;
}

}  // namespace

extern "C" int infini_attn_selftest_timeout(void* stream) {
  unsigned int* status = infini::device_status_word();
  if (!status) return INFINI_ERR_CUDA;
  selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status);
  return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

extern "C" int infini_attn_selftest_approx(const float* x, float* y_poly, float* y_mufu,
                                           unsigned int* bf16_bits, int n, void* stream) {
  if (!x || !y_poly || !y_mufu || !bf16_bits || n < 0) return INFINI_ERR_ARG;
  if (n == 0) return INFINI_OK;
  selftest_kernel<<<(n + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      x, y_poly, y_mufu, bf16_bits, n);
  return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}
