// Tensor-core segment attention for the Infini-attention forward (sm_100a).
//
// One CTA computes one 128-row query tile of one (batch, query head, segment):
//   A_dot = softmax(Q K^T / sqrt(d) + causal mask) V over the segment's keys
//           ("Hugging Face Infini-Attention 再現分析", Local Attention),
//   A_mem = sigma(Q) M_{s-1} / (sigma(Q) z_{s-1}), 0 where the denominator is 0
//           (Memory Retrieval; "Leave No Context Behind" explainer,
//           "メモリの読み出し"),
//   out   = sg(beta_h) A_mem + (1 - sg(beta_h)) A_dot   (Integration),
// reading the memory (M_{s-1} as bf16, z_{s-1} as fp32) that the state scan
// left in the workspace for this segment.
//
// Roles (192 threads):
//   warp 0      TMA producer: Q tile and M_{s-1} once, then the segment's K/V
//               tiles through a two-stage ring.
//   warp 1      allocates TMEM; one thread issues every tcgen05.mma:
//               S_j = Q K_j^T into one of two TMEM score buffers, then
//               O += P_{j-1} V_{j-1} with P read from TMEM, and at the end
//               R = sigma(Q) M_{s-1}.
//   warps 2..5  one thread per query row: online softmax in base 2 (the running
//               max is only raised, and O rescaled, when it grows by more than
//               2^8, so O is rarely touched); writes P (bf16) over its scores;
//               then sigma(Q) in place of Q with the fp32 denominator
//               sigma(q).z, the gate, and the output tile through TMA.
// TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+D), R [256+D, 256+2D).
#include <cuda.h>

#include "kernels.h"
#include "tc_common.cuh"

namespace infini {

namespace {

using namespace tc;

constexpr int kBM = 128;        // query rows per CTA
constexpr int kBN = 128;        // keys per K/V tile
constexpr int kThreads = 192;
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 512;

template <int D>
struct Smem {
  static constexpr int kTile = kBM * D * 2;  // bytes of a 128 x D bf16 tile
  static constexpr int kQ = 0;
  static constexpr int kM = kQ + kTile;
  static constexpr int kK = kM + D * D * 2;
  static constexpr int kV = kK + kStages * kTile;
  static constexpr int kBar = kV + kStages * kTile;
  // barriers: full_k[2], empty_k[2], full_v[2], empty_v[2], s_full[2],
  // p_ready[2], o_done[2], bar_q, bar_m, sq_ready, r_full, drain
  static constexpr int kNumBars = 19;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024
};

struct Bars {
  uint64_t* full_k;
  uint64_t* empty_k;
  uint64_t* full_v;
  uint64_t* empty_v;
  uint64_t* s_full;
  uint64_t* p_ready;
  uint64_t* o_done;  // o_done[b]: P.V of score buffer b complete
  uint64_t* bar_q;
  uint64_t* bar_m;
  uint64_t* sq_ready;
  uint64_t* r_full;
  uint64_t* drain;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
tc_attention(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
             const __grid_constant__ CUtensorMap tm_m, const float* __restrict__ z_pref,
             const float* __restrict__ beta, unsigned int* __restrict__ status, int H_q, int H_kv,
             int L, int S, int T, int tiles_per_seg) {
  using SM = Smem<D>;
  constexpr int kPanels = D / 64;
  constexpr uint32_t kTileBytes = SM::kTile;

  // Tile decode: heaviest query tiles (most key tiles) first; consecutive
  // CTAs take consecutive heads, so the query heads of a KV group run together.
  const int BHq = gridDim.x / (T * tiles_per_seg);
  const int idx = blockIdx.x;
  const int qt = tiles_per_seg - 1 - idx / (T * BHq);
  const int rem = idx % (T * BHq);
  const int s = rem / BHq;
  const int bhq = rem % BHq;
  const int seg0 = s * S;
  const int seg_len = min(S, L - seg0);
  const int q0 = qt * kBM;
  if (q0 >= seg_len) return;  // past the end of a short last segment
  const int n_kv = qt + 1;
  const int b = bhq / H_q, h = bhq % H_q;
  const int g = H_q / H_kv;
  const int bh_kv = b * H_kv + h / g;
  const int BH = (BHq / H_q) * H_kv;
  const int mslice = s * BH + bh_kv;

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = smem + SM::kQ;
  unsigned char* sM = smem + SM::kM;
  unsigned char* sK = smem + SM::kK;
  unsigned char* sV = smem + SM::kV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBar);
  Bars B{bars + 0,  bars + 2,  bars + 4,  bars + 6,  bars + 8,  bars + 10,
         bars + 12, bars + 14, bars + 15, bars + 16, bars + 17, bars + 18};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kTmemSlot);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + SM::kAbort);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&B.full_k[i], 1);
      mbar_init(&B.empty_k[i], 1);
      mbar_init(&B.full_v[i], 1);
      mbar_init(&B.empty_v[i], 1);
      mbar_init(&B.s_full[i], 1);
      mbar_init(&B.p_ready[i], 128);
      mbar_init(&B.o_done[i], 1);
    }
    mbar_init(B.bar_q, 1);
    mbar_init(B.bar_m, 1);
    mbar_init(B.sq_ready, 128);
    mbar_init(B.r_full, 1);
    mbar_init(B.drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_o);
    tma_prefetch_desc(&tm_m);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS[2] = {tmem + 0, tmem + 128};
  const uint32_t tO = tmem + 256;
  const uint32_t tR = tmem + 256 + D;

  const int row_q = seg0 + q0;  // first sequence row of this query tile

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int issued_k = 0, issued_v = 0;
      mbar_arrive_expect_tx(B.bar_q, kTileBytes);
      for (int p = 0; p < kPanels; ++p)
        tma_load_3d(sQ + p * kBM * 128, &tm_q, B.bar_q, p * 64, row_q, bhq);
      mbar_arrive_expect_tx(B.bar_m, D * D * 2);
      for (int p = 0; p < kPanels; ++p)
        tma_load_3d(sM + p * D * 128, &tm_m, B.bar_m, p * 64, 0, mslice);
      for (int j = 0; j < n_kv; ++j) {
        const int st = j & 1;
        const uint32_t par = ((j >> 1) & 1) ^ 1;
        if (!mbar_wait(&B.empty_k[st], par, abort, status)) break;
        mbar_arrive_expect_tx(&B.full_k[st], kTileBytes);
        for (int p = 0; p < kPanels; ++p)
          tma_load_3d(sK + st * kTileBytes + p * kBN * 128, &tm_k, &B.full_k[st], p * 64,
                      seg0 + j * kBN, bh_kv);
        issued_k = j + 1;
        if (!mbar_wait(&B.empty_v[st], par, abort, status)) break;
        mbar_arrive_expect_tx(&B.full_v[st], kTileBytes);
        for (int p = 0; p < kPanels; ++p)
          tma_load_3d(sV + st * kTileBytes + p * kBN * 128, &tm_v, &B.full_v[st], p * 64,
                      seg0 + j * kBN, bh_kv);
        issued_v = j + 1;
      }
      // Before the CTA may exit, every copy issued must have landed.
      mbar_wait(B.bar_q, 0, abort, status, false);
      mbar_wait(B.bar_m, 0, abort, status, false);
      for (int j = (issued_k > 2 ? issued_k - 2 : 0); j < issued_k; ++j)
        mbar_wait(&B.full_k[j & 1], (j >> 1) & 1, abort, status, false);
      for (int j = (issued_v > 2 ? issued_v - 2 : 0); j < issued_v; ++j)
        mbar_wait(&B.full_v[j & 1], (j >> 1) & 1, abort, status, false);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, false, true);
      constexpr uint32_t idesc_ret = idesc_bf16_f32(kBM, D, false, true);
      const uint32_t q_base = smem_u32(sQ), m_base = smem_u32(sM);
      const uint32_t k_base = smem_u32(sK), v_base = smem_u32(sV);
      bool ok = mbar_wait(B.bar_q, 0, abort, status);
      auto issue_pv = [&](int j) -> bool {
        const int st = j & 1;
        const uint32_t par = (j >> 1) & 1;
        if (!mbar_wait(&B.p_ready[st], par, abort, status)) return false;
        if (!mbar_wait(&B.full_v[st], par, abort, status)) return false;
        tc_fence_after();
        const uint32_t vb = v_base + st * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma_ts(tO, tS[st] + kk * 8, sw128_desc(vb + kk * 2048, kBN * 128, 1024), idesc_pv,
                 (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&B.empty_v[st]);
        tc_commit(&B.o_done[st]);
        return true;
      };
      for (int j = 0; ok && j < n_kv; ++j) {
        const int st = j & 1;
        if (!mbar_wait(&B.full_k[st], (j >> 1) & 1, abort, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t kb = k_base + st * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kBM * 128) + (kk & 3) * 32;
          const uint32_t offk = (kk >> 2) * (kBN * 128) + (kk & 3) * 32;
          mma_ss(tS[st], sw128_desc(q_base + off, 16, 1024), sw128_desc(kb + offk, 16, 1024),
                 idesc_qk, kk > 0 ? 1u : 0u);
        }
        tc_commit(&B.s_full[st]);
        tc_commit(&B.empty_k[st]);
        if (j >= 1 && !issue_pv(j - 1)) ok = false;
      }
      if (ok) ok = issue_pv(n_kv - 1);
      if (ok) ok = mbar_wait(B.bar_m, 0, abort, status);
      if (ok) ok = mbar_wait(B.sq_ready, 0, abort, status);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kBM * 128) + (kk & 3) * 32;
          mma_ss(tR, sw128_desc(q_base + off, 16, 1024), sw128_desc(m_base + kk * 2048, D * 128, 1024),
                 idesc_ret, kk > 0 ? 1u : 0u);
        }
        tc_commit(B.r_full);
      }
      // Every MMA issued must be complete before TMEM is released.
      tc_commit(B.drain);
      mbar_wait(B.drain, 0, abort, status, false);
    }
  } else {
    // -------------------------------------------------- softmax / epilogue
    // Waits are made warp-uniform (__all_sync) so that the .sync.aligned
    // TMEM instructions below are always executed by full warps.
    const int r = 32 * (warp & 3) + lane;  // query row within the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int st = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&B.s_full[st], (j >> 1) & 1, abort, status));
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[kBN];
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) tmem_ld32(tS[st] + lane_off + c * 32, sv + c * 32);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < kBN; ++c) sv[c] = __float_as_uint(__uint_as_float(sv[c]) * sl2);
      if (j == qt) {  // diagonal tile: key c is visible to row r iff c <= r
#pragma unroll
        for (int c = 0; c < kBN; ++c)
          if (c > r) sv[c] = __float_as_uint(-INFINITY);
      }
      float mx = __uint_as_float(sv[0]);
#pragma unroll
      for (int c = 1; c < kBN; ++c) mx = fmaxf(mx, __uint_as_float(sv[c]));
      const bool need = mx > m_run + 8.f;
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        // Raise the running max: O (complete through tile j-1) is rescaled.
        const int pj = j - 1;
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&B.o_done[pj & 1], (pj >> 1) & 1, abort, status));
        if (!ok) break;
        tc_fence_after();
        const float f = need ? exp2f(m_run - mx) : 1.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t raw[32];
          tmem_ld32(tO + lane_off + c * 32, raw);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) raw[i] = __float_as_uint(__uint_as_float(raw[i]) * f);
          tmem_st32(tO + lane_off + c * 32, raw);
        }
        tmem_wait_st();
      }
      if (need) {
        l_run *= exp2f(m_run - mx);
        m_run = mx;
      }
      float lsum = 0.f;
#pragma unroll
      for (int c = 0; c < kBN / 64; ++c) {
        uint32_t packed[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p0 = exp2f(__uint_as_float(sv[c * 64 + 2 * i]) - m_run);
          const float p1 = exp2f(__uint_as_float(sv[c * 64 + 2 * i + 1]) - m_run);
          lsum += p0 + p1;
          packed[i] = pack_bf16x2(p0, p1);
        }
        tmem_st32(tS[st] + lane_off + c * 32, packed);
      }
      l_run += lsum;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&B.p_ready[st]);
    }
    // sigma(Q) in place of Q (all QK^T products are complete once the last
    // score tile arrived), and the retrieval denominator sigma(q_r) . z_{s-1}.
    float den = 0.f;
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(B.bar_q, 0, abort, status));
    if (ok) {
      const float* z = z_pref + (size_t)mslice * D;
#pragma unroll 2
      for (int c8 = 0; c8 < D / 8; ++c8) {
        const uint32_t off = sw128_offset(r, c8 * 8, kBM);
        uint4 v = *reinterpret_cast<uint4*>(sQ + off);
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          __nv_bfloat162 pr = *reinterpret_cast<__nv_bfloat162*>(&w[i]);
          const float a = elu1(__low2float(pr));
          const float bb = elu1(__high2float(pr));
          den = fmaf(a, z[c8 * 8 + 2 * i], den);
          den = fmaf(bb, z[c8 * 8 + 2 * i + 1], den);
          w[i] = pack_bf16x2(a, bb);
        }
        *reinterpret_cast<uint4*>(sQ + off) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async();
      mbar_arrive(B.sq_ready);
    }
    if (ok) {
      const int pj = n_kv - 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&B.o_done[pj & 1], (pj >> 1) & 1, abort, status));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(B.r_full, 0, abort, status));
    if (ok) {
      tc_fence_after();
      const float gm = gate_sigmoid(beta[h]);
      const float wo = (1.f - gm) / l_run;
      const float wm = den != 0.f ? gm / den : 0.f;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o_raw[32], r_raw[32];
        tmem_ld32(tO + lane_off + c * 32, o_raw);
        tmem_ld32(tR + lane_off + c * 32, r_raw);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int k0 = i * 8 + 2 * e;
            const float x0 = wo * __uint_as_float(o_raw[k0]) + wm * __uint_as_float(r_raw[k0]);
            const float x1 =
                wo * __uint_as_float(o_raw[k0 + 1]) + wm * __uint_as_float(r_raw[k0 + 1]);
            w[e] = pack_bf16x2(x0, x1);
          }
          *reinterpret_cast<uint4*>(sQ + sw128_offset(r, c * 32 + i * 8, kBM)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      fence_proxy_async();
    }
    tc_fence_before();
    named_barrier(1, 128);  // all four softmax warps, whatever their status
    if (warp == 2 && lane == 0 && *abort == 0) {
      for (int p = 0; p < kPanels; ++p) tma_store_3d(&tm_o, sQ + p * kBM * 128, p * 64, row_q, bhq);
      tma_store_commit();
      tma_store_wait_read();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
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
// 128-byte swizzle, out-of-range rows read as zero.
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
  CUtensorMap tq, tk, tv, to, tm;
  const uint64_t BHq = (uint64_t)p.B * p.H_q, BHkv = (uint64_t)p.B * p.H_kv;
  if (!make_map(&tq, p.q, D, p.L, BHq, kBM) || !make_map(&tk, p.k, D, p.L, BHkv, kBN) ||
      !make_map(&tv, p.v, D, p.L, BHkv, kBN) || !make_map(&to, p.out, D, p.L, BHq, kBM) ||
      !make_map(&tm, p.M_pref, D, D, (uint64_t)p.T * BHkv, D))
    return cudaErrorInvalidValue;
  const int tps = p.S / kBM;
  const long long grid = (long long)BHq * p.T * tps;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const int smem = Smem<D>::kAlloc;
  auto kern = tc_attention<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)grid, kThreads, smem, stream>>>(tq, tk, tv, to, tm, p.z_pref, p.beta, p.status,
                                                   p.H_q, p.H_kv, p.L, p.S, p.T, tps);
  return cudaGetLastError();
}

}  // namespace

bool tc_attention_supported(int d_k, int d_v, int S, bool bf16) {
  return bf16 && d_k == d_v && (d_k == 64 || d_k == 128) && S % kBM == 0;
}

cudaError_t launch_tc_attention(const Problem& p, cudaStream_t stream) {
  if (p.d_k == 128) return launch<128>(p, stream);
  if (p.d_k == 64) return launch<64>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace infini
