// Self-check of the device approximations the tensor-core attention kernel
// uses in place of library functions: the FMA-pipe 2^x (exp2_poly2, both of
// its lanes), the hardware 2^x (ex2.approx), and the bf16 packing of
// probabilities.
#include <cuda_runtime.h>

#include "infini_attn.h"
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

}  // namespace

extern "C" int infini_attn_selftest_approx(const float* x, float* y_poly, float* y_mufu,
                                           unsigned int* bf16_bits, int n, void* stream) {
  if (!x || !y_poly || !y_mufu || !bf16_bits || n < 0) return INFINI_ERR_ARG;
  if (n == 0) return INFINI_OK;
  selftest_kernel<<<(n + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      x, y_poly, y_mufu, bf16_bits, n);
  return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}
