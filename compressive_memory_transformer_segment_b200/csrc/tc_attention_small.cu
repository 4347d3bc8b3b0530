// Tensor-core segment attention for short segments (sm_100a): segment
// length S < 128 with 128 % S == 0 (the 200M-shaped workloads run S = 64).
//
// A CTA takes one 128-row query tile of one (batch, query head); the tile
// covers spt = 128 / S consecutive segments.  For every row r of segment s
// (rows [(s-1)S, sS)):
//   A_dot = softmax(Q K^T / sqrt(d) + mask) V over the keys of the same
//           segment with key <= row ("Hugging Face Infini-Attention 再現分析",
//           Local Attention): the tile's 128 x 128 scores with a
//           block-diagonal causal mask;
//   A_mem = sigma(q_r) M_{s-1} / (sigma(q_r) z_{s-1}), 0 where the denominator
//           is 0 (Memory Retrieval; "Leave No Context Behind" explainer,
//           "メモリの読み出し");
//   out   = sg(beta_h) A_mem + (1 - sg(beta_h)) A_dot   (Integration).
// A row sees at most S <= 64 keys, all in the tile and all in its
// segment's block of the scores, so the softmax is a single pass over that
// block (no running max); P is zero outside it.  The retrieval of every
// segment of the tile is one MMA chain: row r of sigma(Q) sits in the column
// block of its segment of an expanded A operand (zeros elsewhere), and the
// spt memories M_{s-1} are stacked along K as the B operand:
//   R = sigma(Q)_exp [M_{s0-1}; M_{s0}; ...],   O = P V,
//   out_r = g / den_r * R_r + (1 - g) / l_r * O_r   (0 for the first term
//   where den_r = 0).
// The retrieval operand needs only Q and z, so it is built (and R computed)
// while the scores are on the tensor core; the softmax follows.
//
// Roles (160 threads): warp 0 allocates TMEM, lane 0 issues the TMA loads,
// every tcgen05.mma and the output store; warps 1..4 one thread per query
// row (warp w serves TMEM lanes 32 (w % 4) ..).  TMEM: S = [0, 128) (scores,
// then P as bf16 pairs), O = [128, 128 + D), R = [128 + D, 128 + 2D).
#include <cuda.h>

#include "kernels.h"
#include "packed_math.cuh"
#include "pdl.cuh"
#include "tc_common.cuh"

namespace infini {

namespace {

using namespace tc;

constexpr int kBM = 128;  // query rows (and keys) per tile
constexpr int kThreads = 160;
template <int D>
constexpr uint32_t tmem_cols() { return 128 + 2 * D <= 256 ? 256 : 512; }

// Arrival of a whole warp on an mbarrier counted per warp: the warp's
// threads synchronise (ordering their prior writes and TMEM accesses, each
// already fenced as its consumer requires), then one lane arrives.
__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// Shared memory (offsets from a 1024-byte aligned base).
template <int D, int SPT>
struct SmallSmem {
  static constexpr int kTile = kBM * D * 2;          // 128 x D bf16
  static constexpr int kKx = SPT * D;                // K extent of the retrieval MMA
  static constexpr int kQ = 0;                       // Q tile, later the output tile
  static constexpr int kK = kQ + kTile;
  static constexpr int kV = kK + kTile;
  static constexpr int kM = kV + kTile;              // [SPT * D rows][D] bf16, MN-major panels
  static constexpr int kA = kM + kKx * D * 2;        // [128][SPT * D] bf16, K-major panels
  static constexpr int kZ = kA + kBM * kKx * 2;      // z_{s-1} per segment, [SPT][D] fp32
  static constexpr int kBar = kZ + SPT * D * 4;
  // loaded, s_full, p_ready, a_ready, o_full, staged
  static constexpr int kNumBars = 6;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kAlloc = kAbort + 4 + 1024;   // + slack to align the base to 1024
  static_assert(kKx % 64 == 0 && kKx <= 256, "retrieval operand");
  static_assert(kM % 1024 == 0 && kA % 1024 == 0 && kBar % 8 == 0, "alignment");
};

template <int D, int SPT>
__global__ void __launch_bounds__(kThreads, 2)
tc_small_attention(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_m,
                   const __grid_constant__ CUtensorMap tm_o, const float* __restrict__ z_pref,
                   const float* __restrict__ beta, unsigned int* __restrict__ status, int B, int H_q,
                   int H_kv, int L, int T) {
  using SM = SmallSmem<D, SPT>;
  constexpr int S = kBM / SPT;
  constexpr int kPanels = D / 64;
  constexpr int kTileBytes = SM::kTile;

  // ---- the tile: rows [r0, r0 + 128) of (batch b, query head h)
  const int tiles = (L + kBM - 1) / kBM;
  const int tile = blockIdx.x % tiles;
  const int bh = blockIdx.x / tiles;  // b * H_q + h
  const int h = bh % H_q, b = bh / H_q;
  const int h_kv = h / (H_q / H_kv);
  const int r0 = tile * kBM;
  const int s0 = r0 / S;  // first segment of the tile
  const int BHkv = B * H_kv;
  const int bh_kv = b * H_kv + h_kv;

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = smem + SM::kQ;
  unsigned char* sK = smem + SM::kK;
  unsigned char* sV = smem + SM::kV;
  unsigned char* sM = smem + SM::kM;
  unsigned char* sA = smem + SM::kA;
  const float* zs = reinterpret_cast<const float*>(smem + SM::kZ);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBar);
  uint64_t* loaded = bars + 0;
  uint64_t* s_full = bars + 1;
  uint64_t* p_ready = bars + 2;
  uint64_t* a_ready = bars + 3;
  uint64_t* o_full = bars + 4;
  uint64_t* staged = bars + 5;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kTmemSlot);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + SM::kAbort);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // The MMA and copy issue relies on elect.sync picking lane 0 of a
  // converged warp every time (commits and their MMAs from one thread).
  if (__syncthreads_or(elected_lane() != 0)) {
    if (threadIdx.x == 0) atomicOr(status, kStatusLayout);
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(loaded, 1);
    mbar_init(s_full, 1);
    mbar_init(p_ready, 4);  // one arrival per softmax warp
    mbar_init(a_ready, 4);
    mbar_init(o_full, 1);
    mbar_init(staged, 4);
    *abort = 0;
    fence_mbar_init();
  }
  constexpr uint32_t kTmemCols = tmem_cols<D>();
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();
  pdl_wait();  // (nothing above touched global memory)

  if (warp == 0) {
    // ------------------------------------------------ loads, MMAs, store
    // The whole warp runs the sequence and every wait; one elected lane
    // issues.
    if (elect_one()) {
      mbar_arrive_expect_tx(loaded, 3 * kTileBytes + SPT * D * D * 2 + SPT * D * 4);
      for (int p = 0; p < kPanels; ++p) {
        tma_load_3d(sQ + p * kBM * 128, &tm_q, loaded, p * 64, r0, bh);
        tma_load_3d(sK + p * kBM * 128, &tm_k, loaded, p * 64, r0, bh_kv);
        tma_load_3d(sV + p * kBM * 128, &tm_v, loaded, p * 64, r0, bh_kv);
      }
      // M_{s-1} and z_{s-1} of every segment of the tile (a segment past
      // the end of the sequence takes the last one's: its rows are beyond L,
      // and every other row multiplies its block by zero, so it only has to
      // be finite).
      for (int i = 0; i < SPT; ++i) {
        const int s = min(s0 + i, T - 1);
        for (int p = 0; p < kPanels; ++p)
          tma_load_3d(sM + i * D * 128 + p * SPT * D * 128, &tm_m, loaded, p * 64, 0, s * BHkv + bh_kv);
        bulk_load(smem + SM::kZ + i * D * 4, z_pref + (size_t)(s * BHkv + bh_kv) * D, D * 4, loaded);
      }
    }
    bool ok = __all_sync(0xffffffffu, mbar_wait(loaded, 0, abort, status));
    const uint32_t tS = tmem, tO = tmem + 128, tR = tmem + 128 + D;
    if (ok) {
      tc_fence_after();
      if (elect_one()) {
        // S = Q K^T (keys of the whole tile; the mask is applied in the softmax)
        constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBM, false, false);
        const uint64_t dq = sw128_desc(smem_u32(sQ), 16, 1024);
        const uint64_t dk = sw128_desc(smem_u32(sK), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tS, dq + kmajor_step(kk, kBM), dk + kmajor_step(kk, kBM), idesc_qk, kk > 0 ? 1u : 0u);
        tc_commit(s_full);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(a_ready, 0, abort, status));
    }
    if (ok) {
      tc_fence_after();
      if (elect_one()) {
        // R = A_exp [M_{s0-1}; M_{s0}; ...]
        constexpr uint32_t idesc_r = idesc_bf16_f32(kBM, D, false, true);
        const uint64_t da = sw128_desc(smem_u32(sA), 16, 1024);
        const uint64_t dm = sw128_desc(smem_u32(sM), SM::kKx * 128, 1024);
#pragma unroll
        for (int kk = 0; kk < SM::kKx / 16; ++kk)
          mma_ss(tR, da + kmajor_step(kk, kBM), dm + mnmajor_step(kk), idesc_r, kk > 0 ? 1u : 0u);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(p_ready, 0, abort, status));
    }
    if (ok) {
      tc_fence_after();
      if (elect_one()) {
        // O = P V, P read from TMEM (keys 0..63 in columns 0..31, 64..127 in 64..95)
        constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, false, true);
        const uint64_t dv = sw128_desc(smem_u32(sV), kBM * 128, 1024);
#pragma unroll
        for (int kk = 0; kk < kBM / 16; ++kk)
          mma_ts(tO, tS + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8), dv + mnmajor_step(kk), idesc_pv,
                 kk > 0 ? 1u : 0u);
        tc_commit(o_full);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(staged, 0, abort, status));
    }
    if (ok && lane == 0) {
      // Rows past the end of the sequence are clipped by the tensor bounds.
      for (int p = 0; p < kPanels; ++p) tma_store_3d(&tm_o, sQ + p * kBM * 128, p * 64, r0, bh);
      tma_store_commit();
      tma_store_wait_read();  // (the shared-memory source is read; the writes land on their own)
    }
    // Every MMA issued must be complete before TMEM is released (o_full
    // follows all of them; a wait that was abandoned drains here).
    if (!ok && elect_one()) tc_commit(o_full);
    __syncwarp();
    mbar_wait(o_full, 0, abort, status, false);
    __syncwarp();
  } else {
    // ------------------------------------------------ one thread per row
    const int r = 32 * (warp & 3) + lane;  // row of the tile (= TMEM lane)
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tS = tmem + lane_off, tO = tmem + 128 + lane_off, tR = tmem + 128 + D + lane_off;
    const int seg = r / S;                  // the row's segment within the tile
    const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;
    // (The wait on the loads' barrier makes the tiles and z visible here.)
    bool ok = __all_sync(0xffffffffu, mbar_wait(loaded, 0, abort, status));
    float den = 0.f, l = 0.f;
    if (ok) {
      // The retrieval row: sigma(q_r) (bf16) in its segment's column block
      // of the expanded operand, zeros in the other blocks; den_r =
      // sigma(q_r) . z_{s-1} in fp32 on the way.
      const float* z = zs + seg * D;
#pragma unroll 4
      for (int c8 = 0; c8 < D / 8; ++c8) {
        const uint4 v = *reinterpret_cast<const uint4*>(sQ + sw128_offset(r, c8 * 8, kBM));
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
        uint32_t ow[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 sg = pk::sigma_pair(wv[i]);
          den = fmaf(sg.y, z[c8 * 8 + 2 * i + 1], fmaf(sg.x, z[c8 * 8 + 2 * i], den));
          ow[i] = pack_bf16x2(sg.x, sg.y);
        }
#pragma unroll
        for (int blk = 0; blk < SPT; ++blk)
          *reinterpret_cast<uint4*>(sA + sw128_offset(r, blk * D + c8 * 8, kBM)) =
              blk == seg ? make_uint4(ow[0], ow[1], ow[2], ow[3]) : make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async();
      warp_arrive(a_ready);
      ok = __all_sync(0xffffffffu, mbar_wait(s_full, 0, abort, status));
    }
    if (ok) {
      tc_fence_after();
      // Scores of the row's own segment block: keys [seg S, seg S + S),
      // visible up to the row itself.
      uint32_t sv[S];
#pragma unroll
      for (int c = 0; c < S; c += 32) {
        if (S - c >= 32) tmem_ld32(tS + seg * S + c, sv + c);
        else tmem_ld16(tS + seg * S + c, sv + c);
      }
      tmem_wait_ld();
      const int rr = r - seg * S;  // row within the segment
      float m = -INFINITY;
#pragma unroll
      for (int c = 0; c < S; ++c) {
        const float x = c <= rr ? __uint_as_float(sv[c]) * sl2 : -INFINITY;
        sv[c] = __float_as_uint(x);
        m = fmaxf(m, x);
      }
      uint32_t pk[S / 2];
#pragma unroll
      for (int i = 0; i < S / 2; ++i) {
        const float a = ex2_approx(__uint_as_float(sv[2 * i]) - m);
        const float c2 = ex2_approx(__uint_as_float(sv[2 * i + 1]) - m);
        l += a + c2;
        pk[i] = pack_bf16x2(a, c2);
      }
      // P in TMEM: key k of the tile in packed column (k / 64) * 64 +
      // (k % 64) / 2; each 32-column half holds 64 keys, here the row's block
      // and zeros.
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t w32[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          // packed word i of this half holds keys 64 half + 2i, +1
          const int key = 64 * half + 2 * i;
          const int blk = key / S, j = (key % S) / 2;
          w32[i] = blk == seg ? pk[j] : 0u;
        }
        tmem_st32(tS + half * 64, w32);
      }
      tmem_wait_st();
      tc_fence_before();
      warp_arrive(p_ready);
      ok = __all_sync(0xffffffffu, mbar_wait(o_full, 0, abort, status));
    }
    if (ok) {
      tc_fence_after();
      const float gm = gate_sigmoid(__ldg(beta + h));
      // out = g / den R + (1 - g) / l O (the retrieval term 0 where den = 0)
      const float wr = den != 0.f ? gm / den : 0.f;
      const float wo = (1.f - gm) / l;
      // Output row, staged as bf16 in the query tile (whose reads by the
      // tensor core and by this thread are done).
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t o_raw[32], r_raw[32];
        tmem_ld32(tO + c, o_raw);
        tmem_ld32(tR + c, r_raw);
        tmem_wait_ld();
        uint32_t wv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          wv[i] = pack_bf16x2(fmaf(wr, __uint_as_float(r_raw[2 * i]), wo * __uint_as_float(o_raw[2 * i])),
                              fmaf(wr, __uint_as_float(r_raw[2 * i + 1]), wo * __uint_as_float(o_raw[2 * i + 1])));
#pragma unroll
        for (int e = 0; e < 4; ++e)
          *reinterpret_cast<uint4*>(sQ + sw128_offset(r, c + e * 8, kBM)) =
              make_uint4(wv[4 * e], wv[4 * e + 1], wv[4 * e + 2], wv[4 * e + 3]);
      }
      fence_proxy_async();
      warp_arrive(staged);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side

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

// 3-D bf16 map over [planes][rows][cols] (cols contiguous), box 64 x box_rows x 1,
// 128-byte swizzle, out-of-range rows read as zero (and are not written).
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

template <int D, int SPT>
cudaError_t launch(const Problem& p, cudaStream_t stream) {
  CUtensorMap tq, tk, tv, tm, to;
  const uint64_t BHq = (uint64_t)p.B * p.H_q, BHkv = (uint64_t)p.B * p.H_kv;
  if (!make_map(&tq, p.q, D, p.L, BHq, kBM) || !make_map(&tk, p.k, D, p.L, BHkv, kBM) ||
      !make_map(&tv, p.v, D, p.L, BHkv, kBM) || !make_map(&tm, p.M_pref, D, D, (uint64_t)p.T * BHkv, D) ||
      !make_map(&to, p.out, D, p.L, BHq, kBM))
    return cudaErrorInvalidValue;
  const long long grid = (long long)BHq * ((p.L + kBM - 1) / kBM);
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const int smem = SmallSmem<D, SPT>::kAlloc;
  auto kern = tc_small_attention<D, SPT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(true, kern, dim3((unsigned)grid), dim3(kThreads), smem, stream, tq, tk, tv, tm, to,
                    (const float*)p.z_pref, p.beta, p.status, p.B, p.H_q, p.H_kv, p.L, p.T);
}

}  // namespace

bool tc_small_attention_supported(int d_k, int d_v, int S, bool bf16) {
  if (!bf16 || d_k != d_v || (d_k != 64 && d_k != 128) || S < 1 || S >= kBM || kBM % S != 0) return false;
  return (kBM / S) * d_k <= 256 && (kBM / S) * d_k % 64 == 0;
}

cudaError_t launch_tc_small_attention(const Problem& p, cudaStream_t stream) {
  const int spt = kBM / p.S;
  if (p.d_k == 64 && spt == 2) return launch<64, 2>(p, stream);
  if (p.d_k == 64 && spt == 4) return launch<64, 4>(p, stream);
  if (p.d_k == 128 && spt == 2) return launch<128, 2>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace infini
