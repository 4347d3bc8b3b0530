// Tensor-core segment attention for the Infini-attention forward (sm_100a).
//
// For every 128-row query tile of every (batch, query head, segment):
//   A_dot = softmax(Q K^T / sqrt(d) + causal mask) V over the segment's keys
//           ("Hugging Face Infini-Attention 再現分析", Local Attention),
//   A_mem = sigma(Q) M_{s-1} / (sigma(Q) z_{s-1}), 0 where the denominator is 0
//           (Memory Retrieval; "Leave No Context Behind" explainer,
//           "メモリの読み出し"),
//   out   = sg(beta_h) A_mem + (1 - sg(beta_h)) A_dot   (Integration),
// reading the memory (M_{s-1} as bf16, z_{s-1} as fp32) that the state scan
// left in the workspace for this segment.
//
// Persistent kernel, one CTA per SM.  A work item is a PAIR of query tiles
// that read the same keys: two query heads of one KV group at the same tile
// position, or (one query head per KV head) two neighbouring tiles of one
// head.  The pair's two tiles ("slots" A and B) each have their own softmax
// warpgroup and TMEM columns and take turns with the tensor core: while one
// slot's softmax runs, the tensor core computes the other slot's P.V and next
// scores.  Items are taken round-robin (item = CTA + k * grid), ordered by
// (segment, batch row, KV head) group and, inside a group, heaviest first, so
// the CTAs working at any moment share a few groups' keys in L2.
//
// Roles (384 threads, three warpgroups; the first gives registers to the
// other two with setmaxnreg):
//   warp 0      TMA producer: per item K_0, V_0, the two Q tiles, K_1, V_1,
//               ..., then M_{s-1}, through a ring of shared-memory slots; an
//               L2 prefetch of the next item's Q tiles.
//   warp 1      allocates TMEM; one thread issues every tcgen05.mma with the
//               operand descriptors precomputed per group of MMAs:
//               S_j = Q K_j^T, O += P_j V_j (P read from TMEM), and at the end
//               of the item R = sigma(Q) M_{s-1} into the score columns.
//   warps 2, 3  idle.
//   warps 4..7  slot A, warps 8..11 slot B: one thread per query row.  Online
//               softmax in base 2 on the scores in TMEM (row max first, with a
//               three-input max; the running max moves, and O is rescaled,
//               only when the tile max exceeds it by more than 2^8); P (bf16)
//               written over the scores; then sigma(Q) in place of Q with the
//               fp32 retrieval denominator sigma(q).z, and the gated output
//               stored from registers.
// TMEM (512 columns): slot A S = [0, 128), O = [128, 128 + D);
//                     slot B S = [256, 384), O = [384, 384 + D).
#include <cuda.h>

#include "kernels.h"
#include "tc_common.cuh"

namespace infini {

namespace {

using namespace tc;

constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per K/V tile
constexpr int kThreads = 384;
constexpr int kRegsRoles = 104;   // per thread, warpgroup 0 (producer, MMA)
constexpr int kRegsSoftmax = 200; // per thread, warpgroups 1 and 2
constexpr uint32_t kTmemCols = 512;
constexpr int kSmemLimit = 232448;  // opt-in dynamic shared memory per block

template <int D>
struct Smem {
  static constexpr int kTile = kBM * D * 2;  // bytes of a 128 x D bf16 tile (>= D x D for M)
  static constexpr int kRing = (kSmemLimit - 8192 - 2 * kTile) / kTile;
  static constexpr int kQ = 0;  // Q of slot A, Q of slot B
  static constexpr int kRingOff = 2 * kTile;
  static constexpr int kBar = kRingOff + kRing * kTile;
  // ring full[kRing], ring empty[kRing], then two (one per slot) of each of
  // q_full q_empty s_full p_ready sq_ready r_full tmem_free, then z_ready,
  // xbar[4] (one per row quarter) and drain.
  static constexpr int kFull = 0;
  static constexpr int kEmpty = kRing;
  static constexpr int kQFull = 2 * kRing;
  static constexpr int kQEmpty = kQFull + 2;
  static constexpr int kSFull = kQEmpty + 2;
  static constexpr int kPReady = kSFull + 2;
  static constexpr int kSqReady = kPReady + 2;
  static constexpr int kRFull = kSqReady + 2;
  static constexpr int kTFree = kRFull + 2;
  static constexpr int kZReady = kTFree + 2;
  static constexpr int kXBar = kZReady + 1;
  static constexpr int kDrain = kXBar + 4;
  static constexpr int kNumBars = kDrain + 1;
  // z_{s-1} of the item's group, fp32 [D], read as float4: 128-byte aligned.
  static constexpr int kZ = (kBar + kNumBars * 8 + 127) / 128 * 128;
  // Row exchange between the two column halves: fp32 [2 parity][2 half][128 row][2].
  static constexpr int kX = kZ + D * 4;
  static constexpr int kTmemSlot = kX + 2 * 2 * 128 * 2 * 4;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kAlloc = kAbort + 4 + 1024;  // + slack to align the base to 1024
  static_assert(kRing >= 3, "ring too small");
  static_assert(kZ % 16 == 0 && kBar % 8 == 0 && kTmemSlot % 4 == 0, "alignment");
  static_assert(kAlloc <= kSmemLimit, "shared memory");
};

// One work item: a (segment, batch row, KV head) group and two query tiles
// of it (slot x: query head h[x], tile qt[x], n[x] key tiles; n[x] = 0 for
// an empty slot).
struct Item {
  int s, b, h_kv, seg0, seg_len;
  int h[2], qt[2], n[2];
  int n_max;
};

struct Shape {
  int B, H_q, H_kv, L, S, T, g, tps, per_group, items;
};

__device__ __forceinline__ Item decode_item(int idx, const Shape& sh) {
  Item it;
  const int group = idx / sh.per_group;
  const int p = idx - group * sh.per_group;
  it.h_kv = group % sh.H_kv;
  it.b = (group / sh.H_kv) % sh.B;
  it.s = group / (sh.H_kv * sh.B);
  it.seg0 = it.s * sh.S;
  it.seg_len = min(sh.S, sh.L - it.seg0);
  it.n_max = 0;
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    // Tiles of the group in order (query tile descending, then head).
    const int t = 2 * p + x;
    it.h[x] = it.h_kv * sh.g;
    it.qt[x] = 0;
    it.n[x] = 0;
    if (t < sh.g * sh.tps) {
      const int qt = sh.tps - 1 - t / sh.g;
      it.qt[x] = qt;
      it.h[x] = it.h_kv * sh.g + t % sh.g;
      it.n[x] = qt * kBM < it.seg_len ? qt + 1 : 0;
    }
    it.n_max = max(it.n_max, it.n[x]);
  }
  return it;
}

// Arrival of a whole warp on an mbarrier counted per warp: the warp's
// threads synchronise (ordering their prior writes and TMEM accesses, each
// already fenced as its consumer requires), then one lane arrives.
__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// Max of 128 floats (bit patterns in a[64], b[64]) as a shallow tree of
// three-input maxima: 43 + 15 + 5 + 2 + 1 operations, depth 5.
__device__ __forceinline__ float row_max128(const uint32_t* a, const uint32_t* b) {
  auto v = [&](int k) { return __uint_as_float(k < 64 ? a[k] : b[k - 64]); };
  float l1[43];
#pragma unroll
  for (int i = 0; i < 42; ++i) l1[i] = fmax3(v(3 * i), v(3 * i + 1), v(3 * i + 2));
  l1[42] = fmaxf(v(126), v(127));
  float l2[15];
#pragma unroll
  for (int i = 0; i < 14; ++i) l2[i] = fmax3(l1[3 * i], l1[3 * i + 1], l1[3 * i + 2]);
  l2[14] = l1[42];
  float l3[5];
#pragma unroll
  for (int i = 0; i < 5; ++i) l3[i] = fmax3(l2[3 * i], l2[3 * i + 1], l2[3 * i + 2]);
  return fmaxf(fmax3(l3[0], l3[1], l3[2]), fmaxf(l3[3], l3[4]));
}

// P = 2^(s * sl2 - m) for 64 scores (fp32 bit patterns), as 32 bf16 pairs;
// returns the sum of the fp32 values.  Three pairs in four go to the MUFU
// unit, one to the FMA pipe (exp2_poly2), which spreads 2^x over both.
__device__ __forceinline__ float exp_pack64(const uint32_t* sv, float sl2, float m, uint32_t* packed) {
  const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(-m, -m);
  float2 acc2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float2 xx = __ffma2_rn(make_float2(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), sc2, nm2);
    float2 p;
    if ((i & 3) == 3) {
      p = exp2_poly2(xx);
    } else {
      p.x = ex2_approx(xx.x);
      p.y = ex2_approx(xx.y);
    }
    acc2[i & 1] = __fadd2_rn(acc2[i & 1], p);
    packed[i] = pack_bf16x2(p.x, p.y);
  }
  return (acc2[0].x + acc2[0].y) + (acc2[1].x + acc2[1].y);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
tc_attention(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_m,
             const float* __restrict__ z_pref, const float* __restrict__ beta,
             __nv_bfloat16* __restrict__ out, unsigned int* __restrict__ status, const Shape sh) {
  using SM = Smem<D>;
  constexpr int kPanels = D / 64;
  constexpr uint32_t kTileBytes = SM::kTile;
  constexpr int kRing = SM::kRing;

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* ring = smem + SM::kRingOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBar);
  uint64_t* full = bars + SM::kFull;
  uint64_t* empty = bars + SM::kEmpty;
  uint64_t* q_full = bars + SM::kQFull;
  uint64_t* q_empty = bars + SM::kQEmpty;
  uint64_t* s_full = bars + SM::kSFull;
  uint64_t* p_ready = bars + SM::kPReady;
  uint64_t* sq_ready = bars + SM::kSqReady;
  uint64_t* r_full = bars + SM::kRFull;
  uint64_t* tmem_free = bars + SM::kTFree;
  uint64_t* z_ready = bars + SM::kZReady;
  uint64_t* xbars = bars + SM::kXBar;
  uint64_t* drain = bars + SM::kDrain;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kTmemSlot);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + SM::kAbort);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kRing; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(q_full + x, 1);
      mbar_init(q_empty + x, 1);
      mbar_init(s_full + x, 1);
      mbar_init(p_ready + x, 8);  // one arrival per softmax warp
      mbar_init(sq_ready + x, 8);
      mbar_init(r_full + x, 1);
      mbar_init(tmem_free + x, 8);
    }
    mbar_init(z_ready, 8);
    for (int q = 0; q < 4; ++q) mbar_init(xbars + q, 2);
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
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
  const int BHkv = sh.B * sh.H_kv;

  // 384 threads x 168 registers at launch = 4 x 32 x 104 + 8 x 32 x 200; each
  // role's code sits under its own setmaxnreg.
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsRoles));
  if (warp == 0) {
    {
      // ------------------------------------------------ TMA producer
      // The whole warp runs the loop and every wait (kept warp-uniform);
      // lane 0 issues the copies.
      uint32_t rc = 0;                // ring loads issued
      uint32_t qi[2] = {0u, 0u};      // Q loads issued per slot
      bool ok = true;
      auto ring_load = [&](const CUtensorMap* map, int rows_box, int row0, int plane) -> bool {
        const uint32_t slot = rc % kRing, ph = (rc / kRing) & 1u;
        if (!__all_sync(0xffffffffu, mbar_wait(empty + slot, ph ^ 1u, abort, status))) return false;
        if (lane == 0) {
          unsigned char* dst = ring + slot * kTileBytes;
          mbar_arrive_expect_tx(full + slot, (uint32_t)rows_box * D * 2);
          for (int p = 0; p < kPanels; ++p)
            tma_load_3d(dst + p * rows_box * 128, map, full + slot, p * 64, row0, plane);
        }
        ++rc;
        return true;
      };
      for (int idx = blockIdx.x; ok && idx < sh.items; idx += gridDim.x) {
        const Item it = decode_item(idx, sh);
        if (it.n_max == 0) continue;
        const int bh_kv = it.b * sh.H_kv + it.h_kv;
        for (int j = 0; ok && j < it.n_max; ++j) {
          ok = ring_load(&tm_k, kBN, it.seg0 + j * kBN, bh_kv) &&
               ring_load(&tm_v, kBN, it.seg0 + j * kBN, bh_kv);
          if (ok && j == 0) {
            for (int x = 0; ok && x < 2; ++x) {
              if (it.n[x] == 0) continue;
              if (!(ok = __all_sync(0xffffffffu, mbar_wait(q_empty + x, (qi[x] & 1u) ^ 1u, abort, status))))
                break;
              if (lane == 0) {
                unsigned char* dst = smem + SM::kQ + x * kTileBytes;
                mbar_arrive_expect_tx(q_full + x, kTileBytes);
                for (int p = 0; p < kPanels; ++p)
                  tma_load_3d(dst + p * kBM * 128, &tm_q, q_full + x, p * 64, it.seg0 + it.qt[x] * kBM,
                              it.b * sh.H_q + it.h[x]);
              }
              ++qi[x];
            }
          }
        }
        // The next item's query tiles into L2 (the producer runs a few tiles
        // ahead of the tensor core, so they arrive before they are loaded).
        if (ok && lane == 0 && idx + (int)gridDim.x < sh.items) {
          const Item nx = decode_item(idx + gridDim.x, sh);
          for (int x = 0; x < 2; ++x)
            if (nx.n[x] > 0)
              for (int p = 0; p < kPanels; ++p)
                tma_prefetch_l2_3d(&tm_q, p * 64, nx.seg0 + nx.qt[x] * kBM, nx.b * sh.H_q + nx.h[x]);
        }
        // M_{s-1} (D x D, panels of D rows).
        if (ok) ok = ring_load(&tm_m, D, 0, it.s * BHkv + bh_kv);
      }
      // Before the CTA may exit, every copy issued must have landed.
      const uint32_t last = rc < (uint32_t)kRing ? rc : (uint32_t)kRing;
      for (uint32_t i = 0; i < last; ++i) {
        const uint32_t u = rc - 1 - i;
        mbar_wait(full + u % kRing, (u / kRing) & 1u, abort, status, false);
      }
      for (int x = 0; x < 2; ++x)
        if (qi[x] > 0) mbar_wait(q_full + x, (qi[x] - 1) & 1u, abort, status, false);
      __syncwarp();
    }
  } else if (warp == 1) {
    {
      // ------------------------------------------------ MMA issuer
      // The whole warp runs the loop and every wait (kept warp-uniform);
      // lane 0 issues the MMAs and commits.
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, false, true);
      const uint64_t dq[2] = {sw128_desc(smem_u32(smem + SM::kQ), 16, 1024),
                              sw128_desc(smem_u32(smem + SM::kQ + kTileBytes), 16, 1024)};
      const uint64_t dk0 = sw128_desc(smem_u32(ring), 16, 1024);
      const uint64_t dv0 = sw128_desc(smem_u32(ring), kBN * 128, 1024);
      const uint64_t dm0 = sw128_desc(smem_u32(ring), D * 128, 1024);
      uint32_t rc = 0;
      uint32_t pc[2] = {0u, 0u};  // P tiles consumed per slot
      uint32_t ic[2] = {0u, 0u};  // items per slot
      bool ok = true;
      for (int idx = blockIdx.x; ok && idx < sh.items; idx += gridDim.x) {
        const Item it = decode_item(idx, sh);
        if (it.n_max == 0) continue;
        uint32_t ks = 0, kph = 0, vs = 0, vph = 0;
        for (int j = 0; ok && j <= it.n_max; ++j) {
          if (j > 0) {
            vs = rc % kRing;
            vph = (rc / kRing) & 1u;
            ++rc;
          }
          if (j < it.n_max) {
            ks = rc % kRing;
            kph = (rc / kRing) & 1u;
            ++rc;
          }
          const uint64_t dv = dv0 + ((vs * kTileBytes) >> 4);
          const uint64_t dk = dk0 + ((ks * kTileBytes) >> 4);
          bool v_ready = false, k_ready = false;
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            const uint32_t tS = tmem + x * 256, tO = tS + 128;
            if (j > 0 && j - 1 < it.n[x]) {
              // O += P_{j-1} V_{j-1}
              if (!(ok = __all_sync(0xffffffffu, mbar_wait(p_ready + x, pc[x] & 1u, abort, status)))) break;
              ++pc[x];
              if (!v_ready && !(ok = __all_sync(0xffffffffu, mbar_wait(full + vs, vph, abort, status)))) break;
              v_ready = true;
              tc_fence_after();
              if (lane == 0) {
                // P of keys 0..63 sits in columns 0..31, of keys 64..127 in 64..95.
                mma_ts(tO, tS, dv, idesc_pv, j > 1 ? 1u : 0u);
#pragma unroll
                for (int kk = 1; kk < kBN / 16; ++kk)
                  mma_ts(tO, tS + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8), dv + mnmajor_step(kk), idesc_pv, 1u);
              }
            }
            if (j < it.n[x]) {
              // S_j = Q K_j^T
              if (j == 0) {
                // The previous item's epilogue has read this slot's TMEM.
                if (!(ok = __all_sync(0xffffffffu, mbar_wait(tmem_free + x, (ic[x] & 1u) ^ 1u, abort, status)))) break;
                if (!(ok = __all_sync(0xffffffffu, mbar_wait(q_full + x, ic[x] & 1u, abort, status)))) break;
              }
              if (!k_ready && !(ok = __all_sync(0xffffffffu, mbar_wait(full + ks, kph, abort, status)))) break;
              k_ready = true;
              tc_fence_after();
              if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                  mma_ss(tS, dq[x] + kmajor_step(kk, kBM), dk + kmajor_step(kk, kBN), idesc_qk,
                         kk > 0 ? 1u : 0u);
                tc_commit(s_full + x);
              }
            }
          }
          if (!ok) break;
          if (lane == 0) {
            if (j < it.n_max) tc_commit(empty + ks);
            if (j > 0) tc_commit(empty + vs);
          }
        }
        if (!ok) break;
        // Retrieval R = sigma(Q) M_{s-1} into each slot's score columns.
        const uint32_t ms = rc % kRing, mph = (rc / kRing) & 1u;
        ++rc;
        const uint64_t dm = dm0 + ((ms * kTileBytes) >> 4);
        bool m_ready = false;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          if (it.n[x] == 0) continue;
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(sq_ready + x, ic[x] & 1u, abort, status)))) break;
          if (!m_ready && !(ok = __all_sync(0xffffffffu, mbar_wait(full + ms, mph, abort, status)))) break;
          m_ready = true;
          tc_fence_after();
          if (lane == 0) {
            const uint32_t tS = tmem + x * 256;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              mma_ss(tS, dq[x] + kmajor_step(kk, kBM), dm + mnmajor_step(kk), idesc_pv, kk > 0 ? 1u : 0u);
            tc_commit(r_full + x);
            tc_commit(q_empty + x);
          }
        }
        if (!ok) break;
        if (lane == 0) tc_commit(empty + ms);
        for (int x = 0; x < 2; ++x)
          if (it.n[x] > 0) ++ic[x];
      }
      // Every MMA issued must be complete before TMEM is released.
      if (lane == 0) tc_commit(drain);
      __syncwarp();
      mbar_wait(drain, 0, abort, status, false);
      __syncwarp();
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // -------------------------------------------------- softmax / epilogue
    // Warps 4..11 work on every tile of both slots together: warp w owns the
    // rows 32*(w%4) .. +31 (its TMEM lanes) and the column half hc = (w-4)/4
    // (keys 64*hc .. +63 of a score tile, features D/2*hc .. of O and R).
    // The two threads of a row swap their half's tile max (and, at the end
    // of an item, row sum and retrieval denominator) through shared memory,
    // paired by an mbarrier per row quarter.  Waits are made warp-uniform
    // (__all_sync) so that the .sync.aligned TMEM instructions are always
    // executed by full warps.
    const int hc = (warp - 4) >> 2;
    const int qr = warp & 3;
    const int r = 32 * qr + lane;
    const uint32_t lane_off = (uint32_t)(32 * qr) << 16;
    const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;
    float* zs = reinterpret_cast<float*>(smem + SM::kZ);
    float* xb = reinterpret_cast<float*>(smem + SM::kX);
    uint64_t* xbar = xbars + qr;
    // Per-slot state lives in scalars selected by the slot index (the slot
    // loops are not unrolled: one copy of the tile code keeps the hot loop
    // small enough for the instruction cache).
    uint32_t sc0 = 0u, sc1 = 0u, ic0 = 0u, ic1 = 0u, xc = 0u, iz = 0u;
    bool ok = true;
    // Row exchange: post this half's pair of values, later fetch the other's.
    // Slots alternate with the exchange count so that a new post never
    // overwrites a value the partner has not read yet.
    auto xpost = [&](float a, float b) {
      float* mine = xb + (((xc & 1u) * 2 + hc) * 128 + r) * 2;
      mine[0] = a;
      mine[1] = b;
      warp_arrive(xbar);
    };
    auto xget = [&](float& a, float& b) -> bool {
      const bool w_ok = __all_sync(0xffffffffu, mbar_wait(xbar, xc & 1u, abort, status));
      const float* other = xb + (((xc & 1u) * 2 + (hc ^ 1)) * 128 + r) * 2;
      a = other[0];
      b = other[1];
      ++xc;
      return w_ok;
    };
    for (int idx = blockIdx.x; ok && idx < sh.items; idx += gridDim.x) {
      const Item it = decode_item(idx, sh);
      if (it.n_max == 0) continue;
      const int mslice = it.s * BHkv + it.b * sh.H_kv + it.h_kv;
      // z_{s-1} of the group to shared memory (every read of the previous
      // item's copy finished before any thread could get here: those reads
      // precede sq_ready, which the retrieval MMA waited for before r_full).
      {
        const int t = hc * 128 + r;
        if (t < D) zs[t] = __ldg(z_pref + (size_t)mslice * D + t);
        warp_arrive(z_ready);
      }
      float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
#pragma unroll 1
      for (int step = 0; step < 2 * it.n_max; ++step) {
        const int j = step >> 1, x = step & 1;
        if (j >= (x ? it.n[1] : it.n[0])) continue;
        float m_run = x ? m1 : m0, l_run = x ? l1 : l0;
        const uint32_t scx = x ? sc1 : sc0;
        const uint32_t tS = tmem + x * 256 + lane_off;
        ok = __all_sync(0xffffffffu, mbar_wait(s_full + x, scx & 1u, abort, status));
        if (x) sc1 = scx + 1; else sc0 = scx + 1;
        if (!ok) break;
        tc_fence_after();
        // The whole score row (both halves): the tile max is then known to
        // both threads of the row without any exchange; each exponentiates
        // only its own 64 keys.
        uint32_t sv[64], so[64];
        tmem_ld32(tS + 64 * hc, sv);
        tmem_ld32(tS + 64 * hc + 32, sv + 32);
        tmem_ld32(tS + 64 * (hc ^ 1), so);
        tmem_ld32(tS + 64 * (hc ^ 1) + 32, so + 32);
        tmem_wait_ld();
        if (j == (x ? it.qt[1] : it.qt[0])) {
          // Diagonal tile: key c is visible to row r iff c <= r.
          const int lim = r - 64 * hc, limo = r - 64 * (hc ^ 1);
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            if (i > lim) sv[i] = __float_as_uint(-INFINITY);
            if (i > limo) so[i] = __float_as_uint(-INFINITY);
          }
        }
        const float mt = sl2 * row_max128(sv, so);
        if (j == 0) m_run = mt;
        // Exponentials against the running max; after the first tile, if the
        // row's tile max exceeds it by more than 2^8 (rare), rescale this
        // half of O (complete through tile j-1: the scores of tile j were
        // produced after it) and the sum, then take them.  Both threads of
        // the row see the same tile max and decide alike.
        if (j > 0) {
          const bool need = mt > m_run + 8.f;
          if (__any_sync(0xffffffffu, need)) {
            const float f = need ? ex2_approx(m_run - mt) : 1.f;
            const uint32_t tO = tS + 128 + hc * (D / 2);
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              uint32_t raw[16];
              tmem_ld16(tO + c * 16, raw);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 16; ++i) raw[i] = __float_as_uint(__uint_as_float(raw[i]) * f);
              tmem_st16(tO + c * 16, raw);
            }
            tmem_wait_st();
            if (need) {
              l_run *= f;
              m_run = mt;
            }
          }
        }
        uint32_t packed[32];
        const float lsum = exp_pack64(sv, sl2, m_run, packed);
        // P of this half's 64 keys into 32 columns inside its own score
        // columns (keys 0..63 -> columns 0..31, keys 64..127 -> 64..95).
        tmem_st32(tS + 64 * hc, packed);
        l_run += lsum;
        if (x) { m1 = m_run; l1 = l_run; } else { m0 = m_run; l0 = l_run; }
        tmem_wait_st();
        tc_fence_before();
        warp_arrive(p_ready + x);
      }
      if (!ok) break;
      // sigma(Q) in place of Q for this half's features (every QK^T product
      // of the item is complete once its last score tiles arrived) and the
      // partial retrieval denominator sigma(q_r) . z_{s-1} in fp32.
      ok = __all_sync(0xffffffffu, mbar_wait(z_ready, iz & 1u, abort, status));
      ++iz;
      if (!ok) break;
      float den0 = 0.f, den1 = 0.f;
#pragma unroll 1
      for (int x = 0; x < 2; ++x) {
        if ((x ? it.n[1] : it.n[0]) == 0) continue;
        unsigned char* sQ = smem + SM::kQ + x * kTileBytes;
        float den = 0.f;
#pragma unroll 2
        for (int c8 = hc * (D / 16); c8 < (hc + 1) * (D / 16); ++c8) {
          const uint32_t off = sw128_offset(r, c8 * 8, kBM);
          const uint4 v = *reinterpret_cast<const uint4*>(sQ + off);
          const float4 za = reinterpret_cast<const float4*>(zs)[2 * c8];
          const float4 zb = reinterpret_cast<const float4*>(zs)[2 * c8 + 1];
          const float zz[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float a = elu1_fast(bf16lo_to_f32(w[i]));
            const float b = elu1_fast(bf16hi_to_f32(w[i]));
            den = fmaf(a, zz[2 * i], den);
            den = fmaf(b, zz[2 * i + 1], den);
            o[i] = pack_bf16x2(a, b);
          }
          *reinterpret_cast<uint4*>(sQ + off) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        if (x) den1 = den; else den0 = den;
        fence_proxy_async();
        warp_arrive(sq_ready + x);
      }
      // out = (1 - g)/l * O + g/den * R for this half's features: TMEM read
      // out first (then the next item may use the slot's columns), stored
      // from registers.
#pragma unroll 1
      for (int x = 0; x < 2; ++x) {
        if ((x ? it.n[1] : it.n[0]) == 0) continue;
        float lo, dno;
        const float lh = x ? l1 : l0, dh = x ? den1 : den0;
        xpost(lh, dh);
        if (!(ok = xget(lo, dno))) break;
        const float l = lh + lo, dn = dh + dno;
        const uint32_t icx = x ? ic1 : ic0;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(r_full + x, icx & 1u, abort, status)))) break;
        if (x) ic1 = icx + 1; else ic0 = icx + 1;
        tc_fence_after();
        const int hx = x ? it.h[1] : it.h[0], qt = x ? it.qt[1] : it.qt[0];
        const float gm = gate_sigmoid(__ldg(beta + hx));
        const uint32_t tS = tmem + x * 256 + lane_off + hc * (D / 2);
        const uint32_t tO = tmem + x * 256 + lane_off + 128 + hc * (D / 2);
        const float wo = (1.f - gm) / l;
        const float wm = dn != 0.f ? gm / dn : 0.f;
        const float2 wo2 = make_float2(wo, wo), wm2 = make_float2(wm, wm);
        uint32_t w[D / 4];
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          uint32_t o_raw[32], r_raw[32];
          tmem_ld32(tO + c * 32, o_raw);
          tmem_ld32(tS + c * 32, r_raw);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 a = make_float2(__uint_as_float(o_raw[2 * i]), __uint_as_float(o_raw[2 * i + 1]));
            const float2 m = make_float2(__uint_as_float(r_raw[2 * i]), __uint_as_float(r_raw[2 * i + 1]));
            const float2 y = __ffma2_rn(m, wm2, __fmul2_rn(a, wo2));
            w[c * 16 + i] = pack_bf16x2(y.x, y.y);
          }
        }
        tc_fence_before();
        warp_arrive(tmem_free + x);
        if (qt * kBM + r < it.seg_len) {
          uint4* dst = reinterpret_cast<uint4*>(
              out + ((size_t)(it.b * sh.H_q + hx) * sh.L + it.seg0 + qt * kBM + r) * D + hc * (D / 2));
#pragma unroll
          for (int i = 0; i < D / 16; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
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
  CUtensorMap tq, tk, tv, tm;
  const uint64_t BHq = (uint64_t)p.B * p.H_q, BHkv = (uint64_t)p.B * p.H_kv;
  if (!make_map(&tq, p.q, D, p.L, BHq, kBM) || !make_map(&tk, p.k, D, p.L, BHkv, kBN) ||
      !make_map(&tv, p.v, D, p.L, BHkv, kBN) || !make_map(&tm, p.M_pref, D, D, (uint64_t)p.T * BHkv, D))
    return cudaErrorInvalidValue;
  Shape sh;
  sh.B = p.B;
  sh.H_q = p.H_q;
  sh.H_kv = p.H_kv;
  sh.L = p.L;
  sh.S = p.S;
  sh.T = p.T;
  sh.g = p.H_q / p.H_kv;
  sh.tps = p.S / kBM;
  sh.per_group = (sh.g * sh.tps + 1) / 2;
  const long long items = (long long)p.T * BHkv * sh.per_group;
  if (items > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  sh.items = (int)items;
  if (sh.items == 0) return cudaSuccess;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int grid = sh.items < sms ? sh.items : sms;
  const int smem = Smem<D>::kAlloc;
  auto kern = tc_attention<D>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, stream>>>(tq, tk, tv, tm, p.z_pref, p.beta,
                                         static_cast<__nv_bfloat16*>(p.out), p.status, sh);
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
