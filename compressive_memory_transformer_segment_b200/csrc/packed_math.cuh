// Paired fp32 arithmetic (add / mul / fma .f32x2, sm_100) and the ELU+1 map
// on bf16 pairs (the state-scan kernels and the short-segment attention).
// Each half of a paired instruction rounds exactly like the scalar fp32
// instruction.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace infini {
namespace pk {

__device__ __forceinline__ uint64_t as_b64(float2 a) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a.x), "f"(a.y));
  return r;
}
__device__ __forceinline__ float2 as_f2(uint64_t d) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(d));
  return r;
}

// a * b + c per half.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(as_b64(a)), "l"(as_b64(b)), "l"(as_b64(c)));
  return as_f2(d);
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(as_b64(a)), "l"(as_b64(b)));
  return as_f2(d);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(as_b64(a)), "l"(as_b64(b)));
  return as_f2(d);
}

// The two bf16 of a 32-bit word (element 0 in the low half) as floats.
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// sigma(x) = ELU(x) + 1 (x + 1 for x > 0, e^x otherwise) of both halves of a
// bf16 pair, as
//   u = min(x, 0),  sigma = 2^(u log2 e) + (x - u),
// which equals x + 1 (one rounding; 2^0 = 1) for x > 0 and e^x (the hardware
// 2^x approximation, relative error ~2^-22) for x <= 0: the same values as
// the branch form, in fewer instructions (no compare/select, paired add and
// multiply).  An input of -3.39e38 (bf16 0xFF7F) gives exactly 0, which
// masks rows that lie outside the segment.
__device__ __forceinline__ float2 sigma_pair(uint32_t w) {
  const float2 x = bf16x2_to_f2(w);
  const float2 u = make_float2(fminf(x.x, 0.f), fminf(x.y, 0.f));
  const float2 t = mul2(u, make_float2(1.4426950408889634f, 1.4426950408889634f));
  float2 e;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e.x) : "f"(t.x));
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e.y) : "f"(t.y));
  return add2(e, fma2(u, make_float2(-1.f, -1.f), x));
}

// bf16 word of the pair's rounded values (hi) and of the remainders (lo):
// x = hi + lo to ~16 significant bits.
__device__ __forceinline__ void split_pair(float2 x, uint32_t& hi, uint32_t& lo) {
  __nv_bfloat162 h = __floats2bfloat162_rn(x.x, x.y);
  hi = *reinterpret_cast<uint32_t*>(&h);
  const float2 r = fma2(bf16x2_to_f2(hi), make_float2(-1.f, -1.f), x);
  __nv_bfloat162 l = __floats2bfloat162_rn(r.x, r.y);
  lo = *reinterpret_cast<uint32_t*>(&l);
}

}  // namespace pk
}  // namespace infini
