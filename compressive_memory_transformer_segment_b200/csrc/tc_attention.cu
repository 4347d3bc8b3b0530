// Tensor-core segment attention for the Infini-attention forward (sm_100a).
//
// For a 128-row query tile of one (batch, query head, segment):
//   A_dot = softmax(Q K^T / sqrt(d) + causal mask) V over the segment's keys
//           ("Hugging Face Infini-Attention 再現分析", Local Attention),
//   A_mem = sigma(Q) M_{s-1} / (sigma(Q) z_{s-1}), 0 where the denominator is 0
//           (Memory Retrieval; "Leave No Context Behind" explainer,
//           "メモリの読み出し"),
//   out   = sg(beta_h) A_mem + (1 - sg(beta_h)) A_dot   (Integration),
// reading the memory (M_{s-1} as bf16, z_{s-1} as fp32) that the state scan
// left in the workspace for this segment.
//
// Each CTA runs two such query tiles ("slots") that share every K/V tile:
// two query heads of one KV group (grouped-query attention with an even
// group size), otherwise two consecutive query tiles of one head.  The two
// softmax warpgroups alternate with the tensor core: while one turns its
// scores into probabilities, the MMA pipe works on the other slot.
//
// Roles (320 threads):
//   warp 0      TMA producer: both Q tiles and M_{s-1}, then the segment's
//               K/V tiles through a two-stage ring.
//   warp 1      allocates TMEM; one thread issues every tcgen05.mma, with all
//               operand descriptors precomputed (the issuing thread stalls on
//               each MMA until the tensor core takes it, so nothing but
//               descriptor adds sits between consecutive MMAs).
//   warps 2..5  slot 0, warps 6..9 slot 1: one thread per query row.  Online
//               softmax in base 2 on the scores in TMEM (the running max is
//               raised, and O rescaled, only when it grows by more than 2^8);
//               P (bf16) is written over the scores and read by the P.V MMA
//               from TMEM.  At the end: sigma(Q) in place of Q with the fp32
//               denominator sigma(q).z, the gate, and a TMA store of the tile.
// TMEM columns: slot k uses S_k = [256k, 256k+128) (scores, then P, then the
// retrieval sigma(Q) M) and O_k = [256k+128, 256k+128+D).
#include <cuda.h>

#include "kernels.h"
#include "tc_common.cuh"

namespace infini {

namespace {

using namespace tc;

constexpr int kBM = 128;  // query rows per slot
constexpr int kBN = 128;  // keys per K/V tile
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;

template <int D>
struct Smem {
  static constexpr int kTile = kBM * D * 2;  // bytes of a 128 x D bf16 tile
  static constexpr int kQ = 0;               // Q tiles of slot 0 and 1
  static constexpr int kM = kQ + 2 * kTile;
  static constexpr int kK = kM + D * D * 2;
  static constexpr int kV = kK + 2 * kTile;
  static constexpr int kBar = kV + 2 * kTile;
  // full_k[2] empty_k[2] full_v[2] empty_v[2] s_full[2] p_ready[2] o_done[2]
  // sq_ready[2] r_full[2] bar_q bar_m drain
  static constexpr int kNumBars = 21;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kAlloc = kAbort + 4 + 1024;  // + slack to align the base to 1024
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
tc_attention(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
             const __grid_constant__ CUtensorMap tm_m, const float* __restrict__ z_pref,
             const float* __restrict__ beta, unsigned int* __restrict__ status, int B, int H_q,
             int H_kv, int L, int S, int T, int pair_heads) {
  using SM = Smem<D>;
  constexpr int kPanels = D / 64;
  constexpr uint32_t kTileBytes = SM::kTile;

  // ---- work item: group (segment, batch row, KV head), then the pair of slots.
  const int g = H_q / H_kv;
  const int tps = S / kBM;  // query tiles of a full segment
  const int ntp = (tps + 1) / 2;
  const int items = pair_heads ? (g / 2) * tps : g * ntp;
  const int group = blockIdx.x / items;
  const int item = blockIdx.x % items;
  const int h_kv = group % H_kv;
  const int b = (group / H_kv) % B;
  const int s = group / (H_kv * B);
  int h0, h1, qt0, qt1;
  if (pair_heads) {  // heaviest tiles first within the group
    const int qt = tps - 1 - item / (g / 2);
    const int pr = item % (g / 2);
    h0 = h_kv * g + 2 * pr;
    h1 = h0 + 1;
    qt0 = qt1 = qt;
  } else {
    const int tp = ntp - 1 - item / g;
    h0 = h1 = h_kv * g + item % g;
    qt0 = 2 * tp;
    qt1 = 2 * tp + 1;
  }
  const int seg0 = s * S;
  const int seg_len = min(S, L - seg0);
  const bool valid0 = qt0 * kBM < seg_len;
  const bool valid1 = qt1 * kBM < seg_len && qt1 < tps;
  if (!valid0) return;  // slot 0 never starts after slot 1
  const int n_kv0 = qt0 + 1;
  const int n_kv1 = valid1 ? qt1 + 1 : 0;
  const int n_max = max(n_kv0, n_kv1);
  const int bh_kv = b * H_kv + h_kv;
  const int BH = B * H_kv;
  const int mslice = s * BH + bh_kv;

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = smem + SM::kQ;
  unsigned char* sM = smem + SM::kM;
  unsigned char* sK = smem + SM::kK;
  unsigned char* sV = smem + SM::kV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBar);
  uint64_t* full_k = bars + 0;
  uint64_t* empty_k = bars + 2;
  uint64_t* full_v = bars + 4;
  uint64_t* empty_v = bars + 6;
  uint64_t* s_full = bars + 8;
  uint64_t* p_ready = bars + 10;
  uint64_t* o_done = bars + 12;
  uint64_t* sq_ready = bars + 14;
  uint64_t* r_full = bars + 16;
  uint64_t* bar_q = bars + 18;
  uint64_t* bar_m = bars + 19;
  uint64_t* drain = bars + 20;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kTmemSlot);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + SM::kAbort);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&full_k[i], 1);
      mbar_init(&empty_k[i], 1);
      mbar_init(&full_v[i], 1);
      mbar_init(&empty_v[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_ready[i], 128);
      mbar_init(&o_done[i], 1);
      mbar_init(&sq_ready[i], 128);
      mbar_init(&r_full[i], 1);
    }
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
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int issued_k = 0, issued_v = 0;
      mbar_arrive_expect_tx(bar_q, (valid1 ? 2 : 1) * kTileBytes);
      for (int p = 0; p < kPanels; ++p) {
        tma_load_3d(sQ + p * kBM * 128, &tm_q, bar_q, p * 64, seg0 + qt0 * kBM, b * H_q + h0);
        if (valid1)
          tma_load_3d(sQ + kTileBytes + p * kBM * 128, &tm_q, bar_q, p * 64, seg0 + qt1 * kBM,
                      b * H_q + h1);
      }
      mbar_arrive_expect_tx(bar_m, D * D * 2);
      for (int p = 0; p < kPanels; ++p) tma_load_3d(sM + p * D * 128, &tm_m, bar_m, p * 64, 0, mslice);
      for (int j = 0; j < n_max; ++j) {
        const int st = j & 1;
        const uint32_t par = ((j >> 1) & 1) ^ 1;
        if (!mbar_wait(&empty_k[st], par, abort, status)) break;
        mbar_arrive_expect_tx(&full_k[st], kTileBytes);
        for (int p = 0; p < kPanels; ++p)
          tma_load_3d(sK + st * kTileBytes + p * kBN * 128, &tm_k, &full_k[st], p * 64,
                      seg0 + j * kBN, bh_kv);
        issued_k = j + 1;
        if (!mbar_wait(&empty_v[st], par, abort, status)) break;
        mbar_arrive_expect_tx(&full_v[st], kTileBytes);
        for (int p = 0; p < kPanels; ++p)
          tma_load_3d(sV + st * kTileBytes + p * kBN * 128, &tm_v, &full_v[st], p * 64,
                      seg0 + j * kBN, bh_kv);
        issued_v = j + 1;
      }
      // Before the CTA may exit, every copy issued must have landed.
      mbar_wait(bar_q, 0, abort, status, false);
      mbar_wait(bar_m, 0, abort, status, false);
      for (int j = (issued_k > 2 ? issued_k - 2 : 0); j < issued_k; ++j)
        mbar_wait(&full_k[j & 1], (j >> 1) & 1, abort, status, false);
      for (int j = (issued_v > 2 ? issued_v - 2 : 0); j < issued_v; ++j)
        mbar_wait(&full_v[j & 1], (j >> 1) & 1, abort, status, false);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, false, true);
      const uint64_t dq[2] = {sw128_desc(smem_u32(sQ), 16, 1024),
                              sw128_desc(smem_u32(sQ + kTileBytes), 16, 1024)};
      const uint64_t dk[2] = {sw128_desc(smem_u32(sK), 16, 1024),
                              sw128_desc(smem_u32(sK + kTileBytes), 16, 1024)};
      const uint64_t dv[2] = {sw128_desc(smem_u32(sV), kBN * 128, 1024),
                              sw128_desc(smem_u32(sV + kTileBytes), kBN * 128, 1024)};
      const uint64_t dm = sw128_desc(smem_u32(sM), D * 128, 1024);
      const uint32_t tS[2] = {tmem, tmem + 256};
      const uint32_t tO[2] = {tmem + 128, tmem + 256 + 128};
      const int n_kv[2] = {n_kv0, n_kv1};
      auto issue_s = [&](int k, int j) {
        const uint64_t a = dq[k], bk = dk[j & 1];
        const uint32_t d = tS[k];
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(d, a + kmajor_step(kk, kBM), bk + kmajor_step(kk, kBN), idesc_qk, kk > 0 ? 1u : 0u);
        tc_commit(&s_full[k]);
      };
      auto issue_pv = [&](int k, int j) {
        const uint64_t bv = dv[j & 1];
        const uint32_t d = tO[k], a = tS[k];
        const uint32_t acc0 = j > 0 ? 1u : 0u;
        mma_ts(d, a, bv, idesc_pv, acc0);
#pragma unroll
        for (int kk = 1; kk < kBN / 16; ++kk) mma_ts(d, a + kk * 8, bv + mnmajor_step(kk), idesc_pv, 1u);
      };
      bool ok = mbar_wait(bar_q, 0, abort, status) && mbar_wait(&full_k[0], 0, abort, status);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        if (n_kv1 > 0) issue_s(1, 0);
        tc_commit(&empty_k[0]);
      }
      for (int j = 0; ok && j < n_max; ++j) {
        bool v_ready = false, k_ready = false, any_s = false;
        for (int k = 0; k < 2 && ok; ++k) {
          if (j >= n_kv[k]) continue;
          if (!(ok = mbar_wait(&p_ready[k], j & 1, abort, status))) break;
          if (!v_ready) {
            if (!(ok = mbar_wait(&full_v[j & 1], (j >> 1) & 1, abort, status))) break;
            v_ready = true;
          }
          tc_fence_after();
          issue_pv(k, j);
          if (j == n_kv[k] - 1) tc_commit(&o_done[k]);
          if (j + 1 < n_kv[k]) {
            if (!k_ready) {
              if (!(ok = mbar_wait(&full_k[(j + 1) & 1], ((j + 1) >> 1) & 1, abort, status))) break;
              k_ready = true;
              tc_fence_after();
            }
            issue_s(k, j + 1);
            any_s = true;
          }
        }
        if (!ok) break;
        tc_commit(&empty_v[j & 1]);
        if (any_s) tc_commit(&empty_k[(j + 1) & 1]);
      }
      // Retrieval R_k = sigma(Q_k) M_{s-1}, into the slot's score columns.
      constexpr uint32_t idesc_r = idesc_bf16_f32(kBM, D, false, true);
      if (ok) ok = mbar_wait(bar_m, 0, abort, status);
      for (int k = 0; k < 2 && ok; ++k) {
        if (n_kv[k] == 0) continue;
        if (!(ok = mbar_wait(&sq_ready[k], 0, abort, status))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tS[k], dq[k] + kmajor_step(kk, kBM), dm + mnmajor_step(kk), idesc_r, kk > 0 ? 1u : 0u);
        tc_commit(&r_full[k]);
      }
      // Every MMA issued must be complete before TMEM is released.
      tc_commit(drain);
      mbar_wait(drain, 0, abort, status, false);
    }
  } else {
    // -------------------------------------------------- softmax / epilogue
    // Waits are made warp-uniform (__all_sync) so that the .sync.aligned
    // TMEM instructions are always executed by full warps.
    const int k = (warp - 2) >> 2;  // slot
    const bool valid = k == 0 ? true : valid1;
    const int n_kv = k == 0 ? n_kv0 : n_kv1;
    const int qt = k == 0 ? qt0 : qt1;
    const int h = k == 0 ? h0 : h1;
    unsigned char* sQk = sQ + k * kTileBytes;
    const int r = 32 * (warp & 3) + lane;  // query row within the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tS = tmem + 256 * k + lane_off;
    const uint32_t tO = tmem + 256 * k + 128 + lane_off;
    const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = valid;
    for (int j = 0; ok && j < n_kv; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[k], j & 1, abort, status));
      if (!ok) break;
      tc_fence_after();
      // Pass 1: the row max over this tile's scores (on the diagonal tile
      // only keys c <= r count).  The scores stay in TMEM and are read again
      // in pass 2; two 32-column loads are in flight at a time and the
      // reductions use independent accumulators.
      const bool diag = j == qt;
      float mx;
      {
        float m8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) m8[i] = -INFINITY;
#pragma unroll
        for (int c2 = 0; c2 < kBN / 64; ++c2) {
          uint32_t sv[64];
          tmem_ld32(tS + c2 * 64, sv);
          tmem_ld32(tS + c2 * 64 + 32, sv + 32);
          tmem_wait_ld();
          if (diag) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (c2 * 64 + i <= r) m8[i & 7] = fmaxf(m8[i & 7], __uint_as_float(sv[i]));
          } else {
#pragma unroll
            for (int i = 0; i < 64; ++i) m8[i & 7] = fmaxf(m8[i & 7], __uint_as_float(sv[i]));
          }
        }
        mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                   fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      }
      const float mxs = mx * sl2;
      const bool need = mxs > m_run + 8.f;
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        // O holds P.V through tile j-1 (complete: the scores of tile j were
        // produced after it).  Raise the running max and rescale O.
        const float f = need ? exp2f(m_run - mxs) : 1.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t raw[32];
          tmem_ld32(tO + c * 32, raw);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) raw[i] = __float_as_uint(__uint_as_float(raw[i]) * f);
          tmem_st32(tO + c * 32, raw);
        }
        tmem_wait_st();
      }
      if (need) {
        l_run *= exp2f(m_run - mxs);
        m_run = mxs;
      }
      // Pass 2: p = 2^(s * scale - m), row sum, bf16 P over the scores.
      const float nm = -m_run;
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c2 = 0; c2 < kBN / 64; ++c2) {
        uint32_t sv[64], packed[32];
        tmem_ld32(tS + c2 * 64, sv);
        tmem_ld32(tS + c2 * 64 + 32, sv + 32);
        tmem_wait_ld();
        if (diag) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int c0 = c2 * 64 + 2 * i;
            const float p0 = c0 <= r ? ex2_approx(fmaf(__uint_as_float(sv[2 * i]), sl2, nm)) : 0.f;
            const float p1 =
                c0 + 1 <= r ? ex2_approx(fmaf(__uint_as_float(sv[2 * i + 1]), sl2, nm)) : 0.f;
            ls[i & 3] += p0 + p1;
            packed[i] = pack_bf16x2(p0, p1);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float p0 = ex2_approx(fmaf(__uint_as_float(sv[2 * i]), sl2, nm));
            const float p1 = ex2_approx(fmaf(__uint_as_float(sv[2 * i + 1]), sl2, nm));
            ls[i & 3] += p0 + p1;
            packed[i] = pack_bf16x2(p0, p1);
          }
        }
        // P columns 32*c2 .. 32*c2+31 lie inside score columns already read.
        tmem_st32(tS + c2 * 32, packed);
      }
      const float lsum = (ls[0] + ls[1]) + (ls[2] + ls[3]);
      l_run += lsum;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_ready[k]);
    }
    // sigma(Q) in place of Q (every QK^T product of this slot is complete once
    // its last score tile arrived) and the denominator sigma(q_r) . z_{s-1}.
    float den = 0.f;
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_q, 0, abort, status));
    if (ok) {
      const float* z = z_pref + (size_t)mslice * D;
#pragma unroll 2
      for (int c8 = 0; c8 < D / 8; ++c8) {
        const uint32_t off = sw128_offset(r, c8 * 8, kBM);
        uint4 v = *reinterpret_cast<uint4*>(sQk + off);
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
        *reinterpret_cast<uint4*>(sQk + off) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async();
      mbar_arrive(&sq_ready[k]);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&o_done[k], 0, abort, status));
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&r_full[k], 0, abort, status));
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
          *reinterpret_cast<uint4*>(sQk + sw128_offset(r, c * 32 + i * 8, kBM)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      fence_proxy_async();
    }
    if (valid) {
      tc_fence_before();
      named_barrier(1 + k, 128);  // the slot's four warps, whatever their status
      if ((warp & 3) == 2 && lane == 0 && *abort == 0) {
        for (int p = 0; p < kPanels; ++p)
          tma_store_3d(&tm_o, sQk + p * kBM * 128, p * 64, seg0 + qt * kBM, b * H_q + h);
        tma_store_commit();
        tma_store_wait_read();
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
  const int g = p.H_q / p.H_kv;
  const int tps = p.S / kBM;
  const int pair_heads = (g % 2 == 0) ? 1 : 0;
  const long long items = pair_heads ? (long long)(g / 2) * tps : (long long)g * ((tps + 1) / 2);
  const long long grid = (long long)p.T * p.B * p.H_kv * items;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const int smem = Smem<D>::kAlloc;
  auto kern = tc_attention<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)grid, kThreads, smem, stream>>>(tq, tk, tv, to, tm, p.z_pref, p.beta, p.status,
                                                   p.B, p.H_q, p.H_kv, p.L, p.S, p.T, pair_heads);
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
