// Shared device helpers for the Infini-attention kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace infini {

// Bits of the device status word (reported by infini_attn_sync_status).
enum : unsigned int {
  kStatusTimeout = 1u,  // a bounded wait ran out
  kStatusLayout = 2u,   // a kernel found its shared memory not laid out as it requires
};

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// sigma(x) = ELU(x) + 1 (alpha = 1): x + 1 for x > 0, e^x otherwise
// ("Hugging Face Infini-Attention 再現分析", Memory Retrieval).
__device__ __forceinline__ float elu1(float x) { return x > 0.f ? x + 1.f : expf(x); }

// sigma with the hardware 2^x approximation (relative error ~2^-22), for
// operands that are rounded to bf16 right after.
__device__ __forceinline__ float elu1_fast(float x) {
  if (x > 0.f) return x + 1.f;
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x * 1.4426950408889634f));
  return y;
}

// Logistic gate sg(beta); exact 0 / 1 at -inf / +inf.
__device__ __forceinline__ float gate_sigmoid(float b) { return 1.f / (1.f + expf(-b)); }

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

}  // namespace infini
