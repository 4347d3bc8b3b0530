// Tensor-core memory-state scan for the Infini-attention forward (sm_100a).
//
// For one (batch, KV head) chain and one 64-column block of M, the CTA scans
// the segments in order ("Hugging Face Infini-Attention 再現分析", Memory
// Update and State Transfer; "Leave No Context Behind" explainer,
// "メモリの更新" with the delta rule):
//   at the start of segment s it publishes M_{s-1} (bf16, for the attention
//   kernel's retrieval) and z_{s-1} (fp32), then applies the segment's update
//     linear: M += sigma(K)^T V
//     delta : M += sigma(K)^T (V - sigma(K) M_{s-1} / (sigma(K) z_{s-1}))
//     both  : z += sum_t sigma(K_t)
//   and after the last segment writes M_T, z_T (fp32).
//
// Precision.  The update's operands are split into bf16 pairs, x = hi + lo
// with hi = bf16(x) and lo = bf16(x - hi), so the products carry ~16
// significant bits:
//   dM = hi(sK)^T [hi(U) | 1] + lo(sK)^T [hi(U) | 1] + hi(sK)^T lo(U),
// where the constant column of ones yields dz in the same TMEM tile.  TMEM
// accumulates only the current segment's (dM, dz), restarted from zero each
// segment: adding small products into a large running sum inside the tensor
// core loses about one unit in the last place per instruction, which over a
// 1M-token stream exceeds the state tolerance.  The running M and z are fp32
// registers of the math threads (thread t holds row t of M[:, cols] and z[t])
// and take one IEEE fp32 add of (dM, dz) per segment.
// The delta rule's retrieval term R = sigma(K) M_{s-1} uses hi(sK) and a bf16
// snapshot of M_{s-1}; its denominator sigma(K).z_{s-1} is fp32.
//
// Roles (192 threads): warp 0 = TMA producer (K and V blocks of 128 tokens),
// warp 1 = TMEM allocation + the single MMA-issuing thread, warps 2..5 = one
// thread per token (and per row of M).
// TMEM columns: dM|dz accumulator [0, 80) (dM in 0..63, dz in 64), R [128, 192).
#include <cuda.h>

#include "kernels.h"
#include "tc_common.cuh"

namespace infini {

namespace {

using namespace tc;

constexpr int kTok = 128;       // tokens per block
constexpr int kNB = 64;         // columns of M per CTA
constexpr int kNExt = kNB + 16;  // + the z column (padded to an MMA N multiple of 16)
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColR = 128;

template <int D>
struct ScanSmem {
  static constexpr int kK = 0;                       // K block [128][D] (D/64 panels)
  static constexpr int kV = kK + kTok * D * 2;       // V block [128][64]
  static constexpr int kSkHi = kV + kTok * 64 * 2;   // sigma(K) hi [128][128] (2 panels)
  static constexpr int kSkLo = kSkHi + kTok * 128 * 2;
  static constexpr int kUHi = kSkLo + kTok * 128 * 2;  // [U_hi | ones] (2 panels)
  static constexpr int kULo = kUHi + kTok * 128 * 2;   // U_lo (1 panel)
  static constexpr int kMb = kULo + kTok * 64 * 2;     // bf16 M_{s-1}[:, cols] [D][64]
  static constexpr int kZ = kMb + D * 64 * 2;          // fp32 z_{s-1} [128]
  static constexpr int kBar = kZ + 128 * 4;
  // k_full, k_empty, v_full, v_empty, sk_ready, r_ready, u_ready, sk_free,
  // mb_ready, drain
  static constexpr int kNumBars = 10;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kAlloc = kAbort + 4 + 1024;
};

template <int D, bool DELTA>
__global__ void __launch_bounds__(kThreads, 1)
tc_state_scan(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
              const float* __restrict__ M_in, float* __restrict__ M_out, float* __restrict__ z_out,
              float* __restrict__ z_pref, __nv_bfloat16* __restrict__ M_pref,
              unsigned int* __restrict__ status, int L, int S, int T) {
  using SM = ScanSmem<D>;
  const int cb = blockIdx.x;  // column block
  const int c0 = cb * kNB;
  const int bh = blockIdx.y;
  const int BH = gridDim.y;

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sK = smem + SM::kK;
  unsigned char* sV = smem + SM::kV;
  unsigned char* sSkHi = smem + SM::kSkHi;
  unsigned char* sSkLo = smem + SM::kSkLo;
  unsigned char* sUHi = smem + SM::kUHi;
  unsigned char* sULo = smem + SM::kULo;
  unsigned char* sMb = smem + SM::kMb;
  float* zs = reinterpret_cast<float*>(smem + SM::kZ);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBar);
  uint64_t* k_full = bars + 0;
  uint64_t* k_empty = bars + 1;
  uint64_t* v_full = bars + 2;
  uint64_t* v_empty = bars + 3;
  uint64_t* sk_ready = bars + 4;
  uint64_t* r_ready = bars + 5;
  uint64_t* u_ready = bars + 6;
  uint64_t* sk_free = bars + 7;
  uint64_t* mb_ready = bars + 8;
  uint64_t* drain = bars + 9;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kTmemSlot);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + SM::kAbort);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(k_full, 1);
    mbar_init(k_empty, 128);
    mbar_init(v_full, 1);
    mbar_init(v_empty, 128);
    mbar_init(sk_ready, 128);
    mbar_init(r_ready, 1);
    mbar_init(u_ready, 128);
    mbar_init(sk_free, 1);
    mbar_init(mb_ready, 128);
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  // Constant parts of the operand buffers: the ones column of [U_hi | ones]
  // (panel 1, column 0) and, for D = 64, the zero upper half of sigma(K).
  for (int i = threadIdx.x; i < kTok * 64 * 2 / 16; i += kThreads) {
    const int row = i / 8, chunk = i % 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (chunk == (row & 7)) v.x = 0x3F80u;  // element (row, 0) = bf16(1.0)
    *reinterpret_cast<uint4*>(sUHi + kTok * 128 + i * 16) = v;
    if (D == 64) {
      *reinterpret_cast<uint4*>(sSkHi + kTok * 128 + i * 16) = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(sSkLo + kTok * 128 + i * 16) = make_uint4(0, 0, 0, 0);
    }
  }
  fence_proxy_async();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tM = tmem;
  const uint32_t tR = tmem + kColR;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int gb = 0, issued_k = 0, issued_v = 0;
      bool ok = true;
      for (int s = 0; ok && s < T; ++s) {
        const int seg0 = s * S, seg_len = min(S, L - seg0);
        const int nblk = (seg_len + kTok - 1) / kTok;
        for (int tb = 0; tb < nblk; ++tb, ++gb) {
          const uint32_t par = (gb & 1) ^ 1;
          if (!(ok = mbar_wait(k_empty, par, abort, status))) break;
          mbar_arrive_expect_tx(k_full, kTok * D * 2);
          for (int p = 0; p < D / 64; ++p)
            tma_load_3d(sK + p * kTok * 128, &tm_k, k_full, p * 64, seg0 + tb * kTok, bh);
          issued_k = gb + 1;
          if (!(ok = mbar_wait(v_empty, par, abort, status))) break;
          mbar_arrive_expect_tx(v_full, kTok * 64 * 2);
          tma_load_3d(sV, &tm_v, v_full, c0, seg0 + tb * kTok, bh);
          issued_v = gb + 1;
        }
      }
      // Drain: the last copies must have landed before the CTA exits.
      if (issued_k > 0) mbar_wait(k_full, (issued_k - 1) & 1, abort, status, false);
      if (issued_v > 0) mbar_wait(v_full, (issued_v - 1) & 1, abort, status, false);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_r = idesc_bf16_f32(128, kNB, false, true);
      constexpr uint32_t idesc_ext = idesc_bf16_f32(128, kNExt, true, true);
      constexpr uint32_t idesc_lo = idesc_bf16_f32(128, kNB, true, true);
      const uint32_t skhi = smem_u32(sSkHi), sklo = smem_u32(sSkLo);
      const uint32_t uhi = smem_u32(sUHi), ulo = smem_u32(sULo), mb = smem_u32(sMb);
      int gb = 0;
      bool ok = true;
      for (int s = 0; ok && s < T; ++s) {
        const int seg_len = min(S, L - s * S);
        const int nblk = (seg_len + kTok - 1) / kTok;
        if (!(ok = mbar_wait(mb_ready, s & 1, abort, status))) break;
        for (int tb = 0; tb < nblk; ++tb, ++gb) {
          if (!(ok = mbar_wait(sk_ready, gb & 1, abort, status))) break;
          tc_fence_after();
          if (DELTA) {
            // R = hi(sigma(K)) M_{s-1}: tokens x columns, K = D.
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * (kTok * 128) + (kk & 3) * 32;
              mma_ss(tR, sw128_desc(skhi + off, 16, 1024), sw128_desc(mb + kk * 2048, D * 128, 1024),
                     idesc_r, kk > 0 ? 1u : 0u);
            }
            tc_commit(r_ready);
          }
          if (!(ok = mbar_wait(u_ready, gb & 1, abort, status))) break;
          tc_fence_after();
          // dM|dz += sigma(K)^T [U | 1], over the block's 128 tokens.
#pragma unroll
          for (int kk = 0; kk < kTok / 16; ++kk) {
            const uint64_t a_hi = sw128_desc(skhi + kk * 2048, kTok * 128, 1024);
            const uint64_t a_lo = sw128_desc(sklo + kk * 2048, kTok * 128, 1024);
            const uint64_t b_hi = sw128_desc(uhi + kk * 2048, kTok * 128, 1024);
            // The segment's first product restarts the accumulator at zero.
            mma_ss(tM, a_hi, b_hi, idesc_ext, (tb > 0 || kk > 0) ? 1u : 0u);
            mma_ss(tM, a_lo, b_hi, idesc_ext, 1u);
            if (DELTA) mma_ss(tM, a_hi, sw128_desc(ulo + kk * 2048, kTok * 128, 1024), idesc_lo, 1u);
          }
          tc_commit(sk_free);
        }
      }
      tc_commit(drain);
      mbar_wait(drain, 0, abort, status, false);
    }
  } else {
    // -------------------------------------------------- math threads
    const int t = 32 * (warp & 3) + lane;  // token within the block = TMEM lane = row of M
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    bool ok = true;
    // Running state, fp32: row t of M[:, c0..c0+63] and z[t] (rows >= D stay 0).
    float macc[kNB];
    float zacc = 0.f;
#pragma unroll
    for (int i = 0; i < kNB; ++i) macc[i] = t < D ? M_in[((size_t)bh * D + t) * D + c0 + i] : 0.f;
    // z_in was copied to slot 0 of z_pref before this kernel.
    if (t < D) zacc = z_pref[(size_t)bh * D + t];
    int gb = 0;
    for (int s = 0; s <= T && ok; ++s) {
      if (gb > 0) {
        // The previous segment's products are complete: fold (dM, dz) into
        // the running state (this also frees Mb, sigma(K) and U).
        ok = __all_sync(0xffffffffu, mbar_wait(sk_free, (gb - 1) & 1, abort, status));
        if (!ok) break;
        tc_fence_after();
        uint32_t drow[64], dz[32];
        tmem_ld32(tM + lane_off, drow);
        tmem_ld32(tM + lane_off + 32, drow + 32);
        tmem_ld32(tM + lane_off + 64, dz);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < kNB; ++i) macc[i] += __uint_as_float(drow[i]);
        zacc += __uint_as_float(dz[0]);
      }
      if (s == T) {  // final state
        if (t < D) {
          float4* dst = reinterpret_cast<float4*>(M_out + ((size_t)bh * D + t) * D + c0);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            dst[i] = make_float4(macc[4 * i], macc[4 * i + 1], macc[4 * i + 2], macc[4 * i + 3]);
          if (cb == 0) z_out[(size_t)bh * D + t] = zacc;
        }
        break;
      }
      const float zt = zacc;
      if (t < D) {
        uint4* gdst = reinterpret_cast<uint4*>(M_pref + (((size_t)s * BH + bh) * D + t) * D + c0);
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          uint4 v;
          v.x = pack_bf16x2(macc[8 * c8 + 0], macc[8 * c8 + 1]);
          v.y = pack_bf16x2(macc[8 * c8 + 2], macc[8 * c8 + 3]);
          v.z = pack_bf16x2(macc[8 * c8 + 4], macc[8 * c8 + 5]);
          v.w = pack_bf16x2(macc[8 * c8 + 6], macc[8 * c8 + 7]);
          *reinterpret_cast<uint4*>(sMb + sw128_offset(t, 8 * c8, D)) = v;
          gdst[c8] = v;
        }
        if (cb == 0) z_pref[((size_t)s * BH + bh) * D + t] = zt;
      }
      zs[t] = t < D ? zt : 0.f;
      fence_proxy_async();
      mbar_arrive(mb_ready);
      // Every math thread's z entry is in zs before any thread reads it.
      ok = __all_sync(0xffffffffu, mbar_wait(mb_ready, s & 1, abort, status));
      if (!ok) break;

      const int seg0 = s * S, seg_len = min(S, L - seg0);
      const int nblk = (seg_len + kTok - 1) / kTok;
      for (int tb = 0; tb < nblk; ++tb, ++gb) {
        if (tb > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(sk_free, (gb - 1) & 1, abort, status));
          if (!ok) break;
        }
        const bool valid = tb * kTok + t < seg_len;
        // sigma(K) row t as hi/lo bf16 pairs, and r_t = sigma(k_t) . z_{s-1}.
        ok = __all_sync(0xffffffffu, mbar_wait(k_full, gb & 1, abort, status));
        if (!ok) break;
        float r = 0.f;
#pragma unroll 4
        for (int c8 = 0; c8 < D / 8; ++c8) {
          const uint32_t off = sw128_offset(t, 8 * c8, kTok);
          const uint4 kv = *reinterpret_cast<const uint4*>(sK + off);
          const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 pr = *reinterpret_cast<const __nv_bfloat162*>(&kw[i]);
            const float a = valid ? elu1(__low2float(pr)) : 0.f;
            const float b = valid ? elu1(__high2float(pr)) : 0.f;
            r = fmaf(a, zs[8 * c8 + 2 * i], r);
            r = fmaf(b, zs[8 * c8 + 2 * i + 1], r);
            const __nv_bfloat162 hi = __floats2bfloat162_rn(a, b);
            hw[i] = *reinterpret_cast<const uint32_t*>(&hi);
            lw[i] = pack_bf16x2(a - __low2float(hi), b - __high2float(hi));
          }
          *reinterpret_cast<uint4*>(sSkHi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(sSkLo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
        mbar_arrive(k_empty);
        fence_proxy_async();
        mbar_arrive(sk_ready);
        // U = V - R / r (delta) or V (linear), as hi/lo pairs, row t.
        uint32_t rrow[64];
        const float inv_r = r != 0.f ? 1.f / r : 0.f;
        if (DELTA) {
          ok = __all_sync(0xffffffffu, mbar_wait(r_ready, gb & 1, abort, status));
          if (!ok) break;
          tc_fence_after();
          tmem_ld32(tR + lane_off, rrow);
          tmem_ld32(tR + lane_off + 32, rrow + 32);
          tmem_wait_ld();
        }
        ok = __all_sync(0xffffffffu, mbar_wait(v_full, gb & 1, abort, status));
        if (!ok) break;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          const uint32_t off = sw128_offset(t, 8 * c8, kTok);
          const uint4 vv = *reinterpret_cast<const uint4*>(sV + off);
          if (!DELTA) {
            *reinterpret_cast<uint4*>(sUHi + off) = valid ? vv : make_uint4(0, 0, 0, 0);
            continue;
          }
          const uint32_t vw[4] = {vv.x, vv.y, vv.z, vv.w};
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 pr = *reinterpret_cast<const __nv_bfloat162*>(&vw[i]);
            const int c = 8 * c8 + 2 * i;
            float u0 = __low2float(pr) - __uint_as_float(rrow[c]) * inv_r;
            float u1 = __high2float(pr) - __uint_as_float(rrow[c + 1]) * inv_r;
            if (!valid) u0 = u1 = 0.f;
            const __nv_bfloat162 hi = __floats2bfloat162_rn(u0, u1);
            hw[i] = *reinterpret_cast<const uint32_t*>(&hi);
            lw[i] = pack_bf16x2(u0 - __low2float(hi), u1 - __high2float(hi));
          }
          *reinterpret_cast<uint4*>(sUHi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(sULo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
        mbar_arrive(v_empty);
        fence_proxy_async();
        tc_fence_before();
        mbar_arrive(u_ready);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool make_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t planes,
              uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {cols, rows, planes};
  cuuint64_t strides[2] = {cols * 2, cols * rows * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch(const Problem& p, cudaStream_t stream) {
  CUtensorMap tk, tv;
  const uint64_t BHkv = (uint64_t)p.B * p.H_kv;
  if (!make_map(&tk, p.k, D, p.L, BHkv, kTok) || !make_map(&tv, p.v, D, p.L, BHkv, kTok))
    return cudaErrorInvalidValue;
  const int smem = ScanSmem<D>::kAlloc;
  dim3 grid(D / kNB, (unsigned)BHkv);
  auto kern = p.delta ? tc_state_scan<D, true> : tc_state_scan<D, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, stream>>>(tk, tv, p.M_in, p.M_out, p.z_out, p.z_pref,
                                         static_cast<__nv_bfloat16*>(p.M_pref), p.status, p.L,
                                         p.S, p.T);
  return cudaGetLastError();
}

}  // namespace

bool tc_scan_supported(int d_k, int d_v, bool bf16) {
  return bf16 && d_k == d_v && (d_k == 64 || d_k == 128);
}

cudaError_t launch_tc_state_scan(const Problem& p, cudaStream_t stream) {
  if (p.d_k == 128) return launch<128>(p, stream);
  if (p.d_k == 64) return launch<64>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace infini
