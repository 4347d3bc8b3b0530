// Tensor-core segment attention, one query tile per CTA (sm_100a): the
// variant for one query head per KV head, where no two query tiles at the
// same position share keys.  Computes, for one 128-row query tile of one
// (batch, query head, segment):
//   A_dot = softmax(Q K^T / sqrt(d) + causal mask) V over the segment's keys
//           ("Hugging Face Infini-Attention 再現分析", Local Attention),
//   A_mem = sigma(Q) M_{s-1} / (sigma(Q) z_{s-1}), 0 where the denominator is 0
//           (Memory Retrieval; "Leave No Context Behind" explainer,
//           "メモリの読み出し"),
//   out   = sg(beta_h) A_mem + (1 - sg(beta_h)) A_dot   (Integration).
//
// Two CTAs run on every SM (256 TMEM columns, ~97 KB of shared memory for
// d = 128): one CTA's prologue (loads, the first scores) and epilogue
// (retrieval, store) overlap the other's main loop, and the two softmax
// warpgroups take turns with the tensor core.
//
// Roles (192 threads):
//   warp 0      TMA producer: the Q tile, then the segment's K and V tiles one
//               at a time (single buffers), then M_{s-1} into the K buffer.
//               The whole warp runs the loop and waits; lane 0 issues.
//   warp 1      allocates TMEM; lane 0 issues every tcgen05.mma with all
//               operand descriptors precomputed: S_j = Q K_j^T, O += P_j V_j
//               with P read from TMEM, and at the end R = sigma(Q) M_{s-1}.
//   warps 2..5  one thread per query row: the fp32 retrieval denominator
//               sigma(q).z while the first scores are computed; online softmax
//               in base 2 on the scores in TMEM (the running max is raised, and
//               O rescaled, only when it grows by more than 2^8); P (bf16) is
//               written over the scores; at the end sigma(Q) in place of Q,
//               the gate, and a TMA store of the tile.
// TMEM columns: S = [0, 128) (scores, then P, then the retrieval sigma(Q) M)
// and O = [128, 128 + D).
#include <cuda.h>

#include "kernels.h"
#include "tc_common.cuh"

namespace infini {

namespace {

using namespace tc;

constexpr int kBM = 128;  // query rows per CTA
constexpr int kBN = 128;  // keys per K/V tile
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 256;

template <int D>
struct Smem {
  static constexpr int kTile = kBM * D * 2;  // bytes of a 128 x D bf16 tile
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTile;      // K tile, then M_{s-1} (D x D <= 128 x D)
  static constexpr int kV = kK + kTile;
  static constexpr int kBar = kV + kTile;
  // full_k empty_k full_v empty_v s_full p_ready o_done sq_ready r_full bar_q
  // bar_m drain
  static constexpr int kNumBars = 12;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kAlloc = kAbort + 4 + 1024;  // + slack to align the base to 1024
};

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
tc_attention_single(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
             const __grid_constant__ CUtensorMap tm_m, const float* __restrict__ z_pref,
             const float* __restrict__ beta, unsigned int* __restrict__ status, int B, int H_q,
             int H_kv, int L, int S, int T) {
  using SM = Smem<D>;
  constexpr int kPanels = D / 64;
  constexpr uint32_t kTileBytes = SM::kTile;

  // ---- work item: group (segment, batch row, KV head), then (tile, head):
  // the group's tiles run together (L2 reuse of its K/V), heaviest first, and
  // the query heads of a KV group take consecutive CTAs.
  const int g = H_q / H_kv;
  const int tps = S / kBM;
  const int items = g * tps;
  const int group = blockIdx.x / items;
  const int item = blockIdx.x % items;
  const int h_kv = group % H_kv;
  const int b = (group / H_kv) % B;
  const int s = group / (H_kv * B);
  const int qt = tps - 1 - item / g;
  const int h = h_kv * g + item % g;
  const int seg0 = s * S;
  const int seg_len = min(S, L - seg0);
  if (qt * kBM >= seg_len) return;  // past the end of a short last segment
  // The MMA and copy issue relies on elect.sync picking lane 0 of a
  // converged warp every time (commits and their MMAs from one thread).
  if (__syncthreads_or(elected_lane() != 0)) {
    if (threadIdx.x == 0) atomicOr(status, kStatusLayout);
    return;
  }
  const int n_kv = qt + 1;
  const int bh_kv = b * H_kv + h_kv;
  const int BH = B * H_kv;
  const int mslice = s * BH + bh_kv;
  const int row_q = seg0 + qt * kBM;

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = smem + SM::kQ;
  unsigned char* sK = smem + SM::kK;
  unsigned char* sV = smem + SM::kV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBar);
  uint64_t* full_k = bars + 0;
  uint64_t* empty_k = bars + 1;
  uint64_t* full_v = bars + 2;
  uint64_t* empty_v = bars + 3;
  uint64_t* s_full = bars + 4;
  uint64_t* p_ready = bars + 5;
  uint64_t* o_done = bars + 6;
  uint64_t* sq_ready = bars + 7;
  uint64_t* r_full = bars + 8;
  uint64_t* bar_q = bars + 9;
  uint64_t* bar_m = bars + 10;
  uint64_t* drain = bars + 11;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kTmemSlot);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + SM::kAbort);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(full_k, 1);
    mbar_init(empty_k, 1);
    mbar_init(full_v, 1);
    mbar_init(empty_v, 1);
    mbar_init(s_full, 1);
    mbar_init(p_ready, 4);  // one arrival per softmax warp
    mbar_init(o_done, 1);
    mbar_init(sq_ready, 4);
    mbar_init(r_full, 1);
    mbar_init(bar_q, 1);
    mbar_init(bar_m, 1);
    mbar_init(drain, 1);
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

  if (warp == 0) {
    {
      // ------------------------------------------------ TMA producer
      int issued_k = 0, issued_v = 0;
      bool ok = true;
      if (elect_one()) {
        mbar_arrive_expect_tx(bar_q, kTileBytes);
        for (int p = 0; p < kPanels; ++p)
          tma_load_3d(sQ + p * kBM * 128, &tm_q, bar_q, p * 64, row_q, b * H_q + h);
      }
      for (int j = 0; j < n_kv; ++j) {
        const uint32_t par = (j & 1) ^ 1;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(empty_k, par, abort, status)))) break;
        if (elect_one()) {
          mbar_arrive_expect_tx(full_k, kTileBytes);
          for (int p = 0; p < kPanels; ++p)
            tma_load_3d(sK + p * kBN * 128, &tm_k, full_k, p * 64, seg0 + j * kBN, bh_kv);
        }
        issued_k = j + 1;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(empty_v, par, abort, status)))) break;
        if (elect_one()) {
          mbar_arrive_expect_tx(full_v, kTileBytes);
          for (int p = 0; p < kPanels; ++p)
            tma_load_3d(sV + p * kBN * 128, &tm_v, full_v, p * 64, seg0 + j * kBN, bh_kv);
        }
        issued_v = j + 1;
      }
      // M_{s-1} goes into the K buffer once the last score tile is complete.
      bool m_issued = false;
      if (ok && (ok = __all_sync(0xffffffffu, mbar_wait(empty_k, (n_kv & 1) ^ 1, abort, status)))) {
        if (elect_one()) {
          mbar_arrive_expect_tx(bar_m, D * D * 2);
          for (int p = 0; p < kPanels; ++p) tma_load_3d(sK + p * D * 128, &tm_m, bar_m, p * 64, 0, mslice);
        }
        m_issued = true;
      }
      // Before the CTA may exit, every copy issued must have landed.
      mbar_wait(bar_q, 0, abort, status, false);
      if (issued_k > 0) mbar_wait(full_k, (issued_k - 1) & 1, abort, status, false);
      if (issued_v > 0) mbar_wait(full_v, (issued_v - 1) & 1, abort, status, false);
      if (m_issued) mbar_wait(bar_m, 0, abort, status, false);
      __syncwarp();
    }
  } else if (warp == 1) {
    {
      // ------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, false, true);
      constexpr uint32_t idesc_r = idesc_bf16_f32(kBM, D, false, true);
      const uint64_t dq = sw128_desc(smem_u32(sQ), 16, 1024);
      const uint64_t dk = sw128_desc(smem_u32(sK), 16, 1024);
      const uint64_t dv = sw128_desc(smem_u32(sV), kBN * 128, 1024);
      const uint64_t dm = sw128_desc(smem_u32(sK), D * 128, 1024);
      const uint32_t tS = tmem, tO = tmem + 128;
      bool ok = __all_sync(0xffffffffu, mbar_wait(bar_q, 0, abort, status));
      for (int j = 0; ok && j < n_kv; ++j) {
        // S_j = Q K_j^T (the previous P.V has been issued, so P_{j-1} has been
        // read before these MMAs overwrite it: MMAs run in issue order).
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(full_k, j & 1, abort, status)))) break;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(tS, dq + kmajor_step(kk, kBM), dk + kmajor_step(kk, kBN), idesc_qk, kk > 0 ? 1u : 0u);
          tc_commit(s_full);
          tc_commit(empty_k);
        }
        // O += P_j V_j once the softmax has written P_j.
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(p_ready, j & 1, abort, status)))) break;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(full_v, j & 1, abort, status)))) break;
        tc_fence_after();
        if (elect_one()) {
          mma_ts(tO, tS, dv, idesc_pv, j > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 1; kk < kBN / 16; ++kk) mma_ts(tO, tS + kk * 8, dv + mnmajor_step(kk), idesc_pv, 1u);
          tc_commit(empty_v);
        }
      }
      if (ok && elect_one()) tc_commit(o_done);
      // Retrieval R = sigma(Q) M_{s-1}, into the score columns.
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_m, 0, abort, status));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(sq_ready, 0, abort, status));
      if (ok) {
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(tS, dq + kmajor_step(kk, kBM), dm + mnmajor_step(kk), idesc_r, kk > 0 ? 1u : 0u);
          tc_commit(r_full);
        }
      }
      // Every MMA issued must be complete before TMEM is released.
      if (elect_one()) tc_commit(drain);
      __syncwarp();
      mbar_wait(drain, 0, abort, status, false);
      __syncwarp();
    }
  } else {
    // -------------------------------------------------- softmax / epilogue
    // Waits are made warp-uniform (__all_sync) so that the .sync.aligned
    // TMEM instructions are always executed by full warps.
    const int r = 32 * (warp & 3) + lane;  // query row within the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tS = tmem + lane_off;
    const uint32_t tO = tmem + 128 + lane_off;
    const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; ok && j < n_kv; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(s_full, j & 1, abort, status));
      if (!ok) break;
      tc_fence_after();
      // One pass per 64-column half: load the scores, exponentiate against
      // the running max m_run, pack P (bf16) over the scores already read.
      // On the first tile the half's max is taken first (m_run is still
      // -inf); afterwards the max is tracked alongside the exponentials and
      // only checked at the end of the half: if it exceeds m_run by more than
      // 2^8 (rare), the half is recomputed against the new max and O, the row
      // sum and the P half already written are rescaled.
      const bool diag = j == qt;  // key c is visible to row r iff c <= r
      float lsum = 0.f;
#pragma unroll
      for (int hf = 0; hf < kBN / 64; ++hf) {
        uint32_t sv[64];
        tmem_ld32(tS + hf * 64, sv);
        tmem_ld32(tS + hf * 64 + 32, sv + 32);
        tmem_wait_ld();
        if (diag) {
#pragma unroll
          for (int i = 0; i < 64; ++i)
            if (hf * 64 + i > r) sv[i] = __float_as_uint(-INFINITY);
        }
        float mxs;
        if (j == 0 && hf == 0) {
          float m8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) m8[i] = -INFINITY;
#pragma unroll
          for (int i = 0; i < 64; ++i) m8[i & 7] = fmaxf(m8[i & 7], __uint_as_float(sv[i]));
          mxs = sl2 * fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                            fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
          m_run = mxs;
        }
        uint32_t packed[32];
        float2 acc2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        float m8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) m8[i] = -INFINITY;
        {
          const float2 sc = make_float2(sl2, sl2), nm2 = make_float2(-m_run, -m_run);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float s0 = __uint_as_float(sv[2 * i]), s1 = __uint_as_float(sv[2 * i + 1]);
            m8[(2 * i) & 7] = fmaxf(m8[(2 * i) & 7], s0);
            m8[(2 * i + 1) & 7] = fmaxf(m8[(2 * i + 1) & 7], s1);
            const float2 x = __ffma2_rn(make_float2(s0, s1), sc, nm2);
            // One pair in four goes to the FMA pipe (exp2_poly2), the rest to MUFU.
            float2 pp;
            if ((i & 3) == 3) {
              pp = exp2_poly2(x);
            } else {
              pp.x = ex2_approx(x.x);
              pp.y = ex2_approx(x.y);
            }
            const float p0 = pp.x, p1 = pp.y;
            acc2[i & 1] = __fadd2_rn(acc2[i & 1], make_float2(p0, p1));
            packed[i] = pack_bf16x2(p0, p1);
          }
        }
        mxs = sl2 * fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                          fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
        const bool need = mxs > m_run + 8.f;
        if (__any_sync(0xffffffffu, need)) {
          // Rare: the max jumped.  Rescale what was accumulated against the
          // old max and redo this half against the new one.
          const float f = need ? ex2_approx(m_run - mxs) : 1.f;
          if (j > 0) {
            // O holds P.V through tile j-1 (complete: the scores of tile j
            // were produced after it).
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t raw[32];
              tmem_ld32(tO + c * 32, raw);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) raw[i] = __float_as_uint(__uint_as_float(raw[i]) * f);
              tmem_st32(tO + c * 32, raw);
            }
          }
          if (hf > 0) {
            uint32_t pw[32];
            tmem_ld32(tS, pw);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i)
              pw[i] = pack_bf16x2(bf16lo_to_f32(pw[i]) * f, bf16hi_to_f32(pw[i]) * f);
            tmem_st32(tS, pw);
          }
          tmem_wait_st();
          if (need) {
            l_run *= f;
            lsum *= f;
            m_run = mxs;
          }
          const float nm = -m_run;
          acc2[0] = acc2[1] = make_float2(0.f, 0.f);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float p0 = ex2_approx(fmaf(__uint_as_float(sv[2 * i]), sl2, nm));
            const float p1 = ex2_approx(fmaf(__uint_as_float(sv[2 * i + 1]), sl2, nm));
            acc2[i & 1] = __fadd2_rn(acc2[i & 1], make_float2(p0, p1));
            packed[i] = pack_bf16x2(p0, p1);
          }
        }
        lsum += (acc2[0].x + acc2[0].y) + (acc2[1].x + acc2[1].y);
        // P columns 32*hf .. 32*hf+31 lie inside score columns already read.
        tmem_st32(tS + hf * 32, packed);
      }
      l_run += lsum;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_ready);
    }
    // sigma(Q) in place of Q (every QK^T product is complete once the last
    // score tile arrived), and in the same pass the retrieval denominator
    // sigma(q_r) . z_{s-1} in fp32 from the unrounded sigma.  (The wait on
    // the query tile's barrier makes its copy visible to this thread.)
    float den = 0.f;
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_q, 0, abort, status));
    if (ok) {
      const float4* z4 = reinterpret_cast<const float4*>(z_pref + (size_t)mslice * D);
      float dacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
      for (int c8 = 0; c8 < D / 8; ++c8) {
        const uint32_t off = sw128_offset(r, c8 * 8, kBM);
        const uint4 v = *reinterpret_cast<uint4*>(sQ + off);
        const float4 za = __ldg(z4 + 2 * c8), zb = __ldg(z4 + 2 * c8 + 1);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        float sg[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          sg[2 * i] = elu1_fast(bf16lo_to_f32(w[i]));
          sg[2 * i + 1] = elu1_fast(bf16hi_to_f32(w[i]));
        }
        float& a = dacc[c8 & 3];
        a = fmaf(sg[1], za.y, fmaf(sg[0], za.x, a));
        a = fmaf(sg[3], za.w, fmaf(sg[2], za.z, a));
        a = fmaf(sg[5], zb.y, fmaf(sg[4], zb.x, a));
        a = fmaf(sg[7], zb.w, fmaf(sg[6], zb.z, a));
        *reinterpret_cast<uint4*>(sQ + off) =
            make_uint4(pack_bf16x2(sg[0], sg[1]), pack_bf16x2(sg[2], sg[3]), pack_bf16x2(sg[4], sg[5]),
                       pack_bf16x2(sg[6], sg[7]));
      }
      den = (dacc[0] + dacc[1]) + (dacc[2] + dacc[3]);
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(sq_ready);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_done, 0, abort, status));
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(r_full, 0, abort, status));
    if (ok) {
      tc_fence_after();
      const float gm = gate_sigmoid(beta[h]);
      const float wo = (1.f - gm) / l_run;
      const float wm = den != 0.f ? gm / den : 0.f;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o_raw[32], r_raw[32];
        tmem_ld32(tO + c * 32, o_raw);
        tmem_ld32(tS + c * 32, r_raw);
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
    named_barrier(1, 128);  // the four softmax warps, whatever their status
    if (warp == 2 && lane == 0 && *abort == 0) {
      for (int p = 0; p < kPanels; ++p) tma_store_3d(&tm_o, sQ + p * kBM * 128, p * 64, row_q, b * H_q + h);
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
  const long long grid = (long long)p.T * p.B * p.H_q * (p.S / kBM);
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const int smem = Smem<D>::kAlloc;
  auto kern = tc_attention_single<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)grid, kThreads, smem, stream>>>(tq, tk, tv, to, tm, p.z_pref, p.beta, p.status,
                                                   p.B, p.H_q, p.H_kv, p.L, p.S, p.T);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_tc_attention_single(const Problem& p, cudaStream_t stream) {
  if (p.d_k == 128) return launch<128>(p, stream);
  if (p.d_k == 64) return launch<64>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace infini
