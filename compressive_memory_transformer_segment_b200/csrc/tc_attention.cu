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
// position, or, with one query head per KV head, tiles qt and qt - 1 of one
// head (the second skips the first's diagonal key tile).  The pair's two tiles ("slots" A and B) each have their own
// softmax warpgroup and TMEM columns and take turns with the tensor core:
// while one slot's softmax runs, the tensor core computes the other slot's
// P.V and next scores.  Items are ordered by (segment, batch row, KV head)
// group and, inside a group, heaviest first; they are handed out round-robin
// in units of two, an item and its mirror image in the group's order
// (heaviest with lightest), so that every unit costs the same and the CTAs,
// which work on a few neighbouring groups at any moment, share those groups'
// keys in L2.  (With one query head per KV head and d = 64 the
// one-tile-per-CTA kernel runs instead.)
//
// Roles (384 threads, three warpgroups; the first gives registers to the
// other two with setmaxnreg):
//   warp 0      TMA producer: per item K_0, V_0, K_1, V_1, ..., M_{s-1}
//               through a ring of shared-memory slots, and, early in the
//               item, the next item's two query tiles (double-buffered), each
//               with its z_{s-1} (a bulk copy on the tile's barrier).
//   warp 1      allocates TMEM; one thread issues every tcgen05.mma:
//               S_j = Q K_j^T, O += P_j V_j (P read from TMEM), and at the end
//               of the item R' = (sigma(Q) c) M_{s-1} into O, then the next
//               item's first S.  A slot's P.V and next QK^T go back to back.
//   warps 2, 3  idle.
//   warps 4..7  slot A, warps 8..11 slot B: one thread per query row.  Online
//               softmax in base 2 on the scores in TMEM (the first tile's row
//               max is the reference; it moves, and O is rescaled, only when
//               a tile's sum exceeds 2^16); P (bf16) written over the scores;
//               the retrieval denominator sigma(q).z while the tensor core
//               works on the first tile; at the end the retrieval rows
//               sigma(Q) c in place of Q (the retrieval is folded into O, see
//               the epilogue), the read-out of O, and one TMA store of the
//               output tile staged in the query tile's buffer.
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
// Registers per thread after setmaxnreg: 384 x 168 at launch =
// 128 x kRegsRoles + 256 x kRegsSoftmax.
constexpr int kRegsRoles = 104;    // warpgroup 0 (producer, MMA)
constexpr int kRegsSoftmax = 200;  // warpgroups 1 and 2
static_assert(128 * kRegsRoles + 256 * kRegsSoftmax <= kThreads * 168, "registers");
constexpr uint32_t kTmemCols = 512;
constexpr int kSmemLimit = 232448;  // opt-in dynamic shared memory per block

template <int D>
struct Smem {
  static constexpr int kTile = kBM * D * 2;  // bytes of a 128 x D bf16 tile (>= D x D for M)
  // Q tiles: [slot][item parity] (the next item's Q loads during this one).
  static constexpr int kRing = (kSmemLimit - 3072 - 4 * kTile) / kTile;
  static constexpr int kQ = 0;
  static constexpr int kRingOff = 4 * kTile;
  static constexpr int kBar = kRingOff + kRing * kTile;
  // ring full[kRing], ring empty[kRing], q_full[4] q_empty[4] (per Q tile,
  // with its z), then two (one per slot) of each of s_full p_ready sq_ready
  // r_full tmem_free o_staged, then drain.
  static constexpr int kFull = 0;
  static constexpr int kEmpty = kRing;
  static constexpr int kQFull = 2 * kRing;
  static constexpr int kQEmpty = kQFull + 4;
  static constexpr int kSFull = kQEmpty + 4;
  static constexpr int kPReady = kSFull + 2;
  static constexpr int kSqReady = kPReady + 2;
  static constexpr int kRFull = kSqReady + 2;
  static constexpr int kTFree = kRFull + 2;
  static constexpr int kOStaged = kTFree + 2;
  static constexpr int kDrain = kOStaged + 2;
  static constexpr int kNumBars = kDrain + 1;
  // z_{s-1} per query tile, fp32 [4][D] (copied in with the tile), read as
  // float4: 128-byte aligned.
  static constexpr int kZ = (kBar + kNumBars * 8 + 127) / 128 * 128;
  static constexpr int kTmemSlot = kZ + 4 * D * 4;
  static constexpr int kAbort = kTmemSlot + 4;
  // The dynamic shared memory base is 1024-byte aligned (checked at entry).
  static constexpr int kAlloc = kAbort + 4;
  static_assert(kRing >= 3, "ring too small");
  static_assert(kZ % 16 == 0 && kBar % 8 == 0 && kTmemSlot % 4 == 0, "alignment");
  static_assert(kAlloc <= kSmemLimit, "shared memory");
};

// One work item: a (segment, batch row, KV head) group and two query tiles
// of it (slot x: query head h[x], tile qt[x], n[x] key tiles; n[x] = 0 for
// an empty slot).  Both slots read key tiles 0 .. n_max - 1.
struct Item {
  int s, b, h_kv, seg0, seg_len;
  int h[2], qt[2], n[2];
  int n_max;
};

// n / d for 0 <= n < 2^31 as a multiply and a shift: m = ceil(2^(31 + l) / d),
// l = ceil(log2 d) (exact there: the rounding error of m stays below one
// step of n / d).
struct FastDiv {
  uint32_t m, sh;
};
__host__ __device__ inline FastDiv make_fastdiv(uint32_t d) {
  uint32_t l = 0;
  while ((1ull << l) < d) ++l;
  return FastDiv{(uint32_t)(((1ull << (31 + l)) + d - 1) / d), 31 + l};
}
__device__ __forceinline__ int fdiv(int n, FastDiv f) {
  return (int)(((unsigned long long)(uint32_t)n * f.m) >> f.sh);
}

struct Shape {
  int B, H_q, H_kv, L, S, T, g, tps, per_group, upg, units;
  FastDiv by_per_group, by_upg, by_H_kv, by_B;
};

__device__ __forceinline__ Item decode_item(int idx, const Shape& sh) {
  Item it;
  const int group = fdiv(idx, sh.by_per_group);
  const int p = idx - group * sh.per_group;
  const int gb = fdiv(group, sh.by_H_kv);  // group / H_kv
  it.h_kv = group - gb * sh.H_kv;
  it.s = fdiv(gb, sh.by_B);
  it.b = gb - it.s * sh.B;
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

// The CTA's k-th item.  Work is handed out in units, round-robin (unit =
// CTA + (k / 2) * grid); a unit is the item at position r of its group and
// the item at the mirrored position per_group - 1 - r (empty when the two
// coincide).  Positions run from the heaviest item to the lightest, so every
// unit holds about the same number of key tiles (tps + 1 when every tile is
// full) and the CTAs finish together.
__device__ __forceinline__ bool seq_valid(int k, const Shape& sh) {
  return (int)blockIdx.x + (k >> 1) * (int)gridDim.x < sh.units;
}

__device__ __forceinline__ Item seq_item(int k, const Shape& sh) {
  const int u = (int)blockIdx.x + (k >> 1) * (int)gridDim.x;
  const int group = fdiv(u, sh.by_upg), r = u - group * sh.upg;
  const int p = (k & 1) ? sh.per_group - 1 - r : r;
  if ((k & 1) && p == r) {
    Item it;
    it.s = it.b = it.h_kv = it.seg0 = it.seg_len = 0;
    it.h[0] = it.h[1] = it.qt[0] = it.qt[1] = 0;
    it.n[0] = it.n[1] = 0;
    it.n_max = 0;
    return it;
  }
  return decode_item(group * sh.per_group + p, sh);
}

// Arrival of a whole warp on an mbarrier counted per warp: the warp's
// threads synchronise (ordering their prior writes and TMEM accesses, each
// already fenced as its consumer requires), then one lane arrives.
__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// Max of 128 floats (bit patterns in a[64], b[64]) with three-input maxima:
// 16 independent accumulators over 8 values each (depth 4), then a short
// tree; few values live at once.
__device__ __forceinline__ float row_max128(const uint32_t* a, const uint32_t* b) {
  auto v = [&](int k) { return __uint_as_float(k < 64 ? a[k] : b[k - 64]); };
  float acc[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) acc[k] = fmax3(v(k), v(16 + k), v(32 + k));
#pragma unroll
  for (int k = 0; k < 16; ++k) acc[k] = fmax3(acc[k], v(48 + k), v(64 + k));
#pragma unroll
  for (int k = 0; k < 16; ++k) acc[k] = fmax3(acc[k], v(80 + k), v(96 + k));
#pragma unroll
  for (int k = 0; k < 16; ++k) acc[k] = fmaxf(acc[k], v(112 + k));
  float t[6];
#pragma unroll
  for (int i = 0; i < 5; ++i) t[i] = fmax3(acc[3 * i], acc[3 * i + 1], acc[3 * i + 2]);
  t[5] = acc[15];
  return fmaxf(fmax3(t[0], t[1], t[2]), fmax3(t[3], t[4], t[5]));
}

// P = 2^(s * sl2 - m) for 64 scores (fp32 bit patterns), as 32 bf16 pairs;
// returns the sum of the fp32 values.  Three pairs in four go to the MUFU
// unit, one to the FMA pipe (exp2_poly2), which spreads 2^x over both.
// MASKED (a diagonal tile, whose masked scores are -inf): masked keys get
// exactly 0 on both pipes.
template <bool MASKED>
__device__ __forceinline__ float exp_pack64(const uint32_t* sv, float sl2, float m, uint32_t* packed) {
  const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(-m, -m);
  float2 acc2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float2 xx = __ffma2_rn(make_float2(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), sc2, nm2);
    float2 p;
    if ((i & 3) == 3) {
      p = exp2_poly2<MASKED>(xx);
    } else {
      p.x = ex2_approx(xx.x);
      p.y = ex2_approx(xx.y);
    }
    acc2[i & 1] = __fadd2_rn(acc2[i & 1], p);
    packed[i] = pack_bf16x2(p.x, p.y);
  }
  return (acc2[0].x + acc2[0].y) + (acc2[1].x + acc2[1].y);
}

// sigma(x) = x + 1 (x > 0), e^x (x <= 0) of a bf16 pair, in fp32; e^x as
// 2^(x log2 e) on the MUFU unit (which measured faster here than sharing the
// work with the FMA pipe: the end of an item has no MUFU-heavy softmax
// running beside it).
__device__ __forceinline__ float2 sigma2(uint32_t w) {
  const float2 xv = make_float2(bf16lo_to_f32(w), bf16hi_to_f32(w));
  const float ex = ex2_approx(xv.x * 1.4426950408889634f), ey = ex2_approx(xv.y * 1.4426950408889634f);
  return make_float2(xv.x > 0.f ? xv.x + 1.f : ex, xv.y > 0.f ? xv.y + 1.f : ey);
}

// sigma(q_r) of row r of a 128-row query tile in shared memory, into sg[D]
// (fp32, unrounded), and the retrieval denominator sigma(q_r) . z_{s-1}
// (z in shared memory, read as float4), in one pass over the row.
template <int D>
__device__ __forceinline__ float sigma_row(const unsigned char* sQ, int r, const float* zs, float* sg) {
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int c8 = 0; c8 < D / 8; ++c8) {
    const uint4 v = *reinterpret_cast<const uint4*>(sQ + sw128_offset(r, c8 * 8, kBM));
    const float4 za = reinterpret_cast<const float4*>(zs)[2 * c8];
    const float4 zb = reinterpret_cast<const float4*>(zs)[2 * c8 + 1];
    const float2 s0 = sigma2(v.x), s1 = sigma2(v.y), s2 = sigma2(v.z), s3 = sigma2(v.w);
    float* o = sg + c8 * 8;
    o[0] = s0.x; o[1] = s0.y; o[2] = s1.x; o[3] = s1.y;
    o[4] = s2.x; o[5] = s2.y; o[6] = s3.x; o[7] = s3.y;
    float& a = acc[c8 & 3];
    a = fmaf(s0.y, za.y, fmaf(s0.x, za.x, a));
    a = fmaf(s1.y, za.w, fmaf(s1.x, za.z, a));
    a = fmaf(s2.y, zb.y, fmaf(s2.x, zb.x, a));
    a = fmaf(s3.y, zb.w, fmaf(s3.x, zb.z, a));
  }
  return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// Row r of the query tile replaced, in place, by bf16(sg * c).
template <int D>
__device__ __forceinline__ void store_scaled_row(unsigned char* sQ, int r, const float* sg, float c) {
#pragma unroll
  for (int c8 = 0; c8 < D / 8; ++c8) {
    const float* v = sg + c8 * 8;
    *reinterpret_cast<uint4*>(sQ + sw128_offset(r, c8 * 8, kBM)) =
        make_uint4(pack_bf16x2(v[0] * c, v[1] * c), pack_bf16x2(v[2] * c, v[3] * c),
                   pack_bf16x2(v[4] * c, v[5] * c), pack_bf16x2(v[6] * c, v[7] * c));
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
tc_attention(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_m,
             const __grid_constant__ CUtensorMap tm_o, const float* __restrict__ z_pref,
             const float* __restrict__ beta, unsigned int* __restrict__ status, const Shape sh) {
  using SM = Smem<D>;
  constexpr int kPanels = D / 64;
  constexpr uint32_t kTileBytes = SM::kTile;
  constexpr int kRing = SM::kRing;

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // The swizzled tiles need 1024-byte aligned addresses; the layout fills
  // the opt-in maximum, leaving no room to realign.  The MMA and copy issue
  // relies on elect.sync picking lane 0 of a converged warp every time
  // (commits and their MMAs from one thread).  Either failing, the CTA
  // computes nothing (the decision is the same for every thread).
  const bool misplaced = (smem_u32(smem_raw) & 1023u) != 0 || elected_lane() != 0;
  if (__syncthreads_or(misplaced)) {
    if (threadIdx.x == 0) atomicOr(status, kStatusLayout);
    return;
  }
  unsigned char* smem = smem_raw;
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
  uint64_t* o_staged = bars + SM::kOStaged;
  uint64_t* drain = bars + SM::kDrain;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kTmemSlot);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + SM::kAbort);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kRing; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    for (int b = 0; b < 4; ++b) {
      mbar_init(q_full + b, 1);
      mbar_init(q_empty + b, 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(s_full + x, 1);
      mbar_init(p_ready + x, 4);  // one arrival per softmax warp of the slot
      mbar_init(sq_ready + x, 4);
      mbar_init(r_full + x, 1);
      mbar_init(tmem_free + x, 4);
      mbar_init(o_staged + x, 4);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_m);
    tma_prefetch_desc(&tm_o);
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

  // Each role's code sits under its own setmaxnreg (register split above).
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsRoles));
  if (warp == 0) {
    {
      // ------------------------------------------------ TMA producer
      // The whole warp runs the loop and every wait (kept warp-uniform);
      // lane 0 issues the copies.  Ring entries per item: K_0 V_0 K_1 V_1
      // ... M_{s-1}.
      uint32_t rc = 0;                // ring loads issued
      uint32_t qi[2] = {0u, 0u};      // Q loads issued per slot (tile = 2 * slot + count % 2)
      bool ok = true;
      auto ring_load = [&](const CUtensorMap* map, int rows_box, int row0, int plane) -> bool {
        const uint32_t slot = rc % kRing, ph = (rc / kRing) & 1u;
        if (!__all_sync(0xffffffffu, mbar_wait(empty + slot, ph ^ 1u, abort, status))) return false;
        if (elect_one()) {
          unsigned char* dst = ring + slot * kTileBytes;
          mbar_arrive_expect_tx(full + slot, (uint32_t)rows_box * D * 2);
          for (int p = 0; p < kPanels; ++p)
            tma_load_3d(dst + p * rows_box * 128, map, full + slot, p * 64, row0, plane);
        }
        ++rc;
        return true;
      };
      // Query tiles of an item into the slots' next Q tiles, each with the
      // item's z_{s-1} (D floats) in the tile's z buffer.  A tile is free
      // once the output store of the item two back (which staged its output
      // there) has read it; the softmax warps signal that after the first
      // scores of the item in between.
      auto q_load = [&](const Item& nx) -> bool {
        for (int x = 0; x < 2; ++x) {
          if (nx.n[x] == 0) continue;
          const uint32_t b = 2 * x + (qi[x] & 1u);
          if (!__all_sync(0xffffffffu, mbar_wait(q_empty + b, ((qi[x] >> 1) & 1u) ^ 1u, abort, status)))
            return false;
          if (elect_one()) {
            unsigned char* dst = smem + SM::kQ + b * kTileBytes;
            mbar_arrive_expect_tx(q_full + b, kTileBytes + D * 4);
            for (int p = 0; p < kPanels; ++p)
              tma_load_3d(dst + p * kBM * 128, &tm_q, q_full + b, p * 64, nx.seg0 + nx.qt[x] * kBM,
                          nx.b * sh.H_q + nx.h[x]);
            bulk_load(smem + SM::kZ + b * D * 4,
                      z_pref + (size_t)(nx.s * BHkv + nx.b * sh.H_kv + nx.h_kv) * D, D * 4, q_full + b);
          }
          ++qi[x];
        }
        return true;
      };
      if (seq_valid(0, sh)) ok = q_load(seq_item(0, sh));
      for (int k = 0; ok && seq_valid(k, sh); ++k) {
        const Item it = seq_item(k, sh);
        const bool has_next = seq_valid(k + 1, sh);
        if (it.n_max == 0) {
          // An empty item (past the end of a short last segment, or the
          // missing half of a unit) still hands on the next item's query tiles.
          if (has_next) ok = q_load(seq_item(k + 1, sh));
          continue;
        }
        const int bh_kv = it.b * sh.H_kv + it.h_kv;
        for (int j = 0; ok && j < it.n_max; ++j) {
          ok = ring_load(&tm_k, kBN, it.seg0 + j * kBN, bh_kv) &&
               ring_load(&tm_v, kBN, it.seg0 + j * kBN, bh_kv);
          // The next item's query tiles, after this item's second key tile
          // (or its only one).
          if (ok && j == min(1, it.n_max - 1) && has_next) ok = q_load(seq_item(k + 1, sh));
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
        for (int p = 0; p < 2; ++p) {
          const uint32_t uses = (qi[x] + 1u - p) / 2u;  // loads into tile 2x + p
          if (uses > 0) mbar_wait(q_full + 2 * x + p, (uses - 1) & 1u, abort, status, false);
        }
      __syncwarp();
    }
  } else if (warp == 1) {
    {
      // ------------------------------------------------ MMA issuer
      // The whole warp runs the loop and every wait (kept warp-uniform);
      // lane 0 issues the MMAs and commits.
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, false, true);
      const uint64_t dq0 = sw128_desc(smem_u32(smem + SM::kQ), 16, 1024);
      const uint64_t dk0 = sw128_desc(smem_u32(ring), 16, 1024);
      const uint64_t dv0 = sw128_desc(smem_u32(ring), kBN * 128, 1024);
      const uint64_t dm0 = sw128_desc(smem_u32(ring), D * 128, 1024);
      uint32_t base = 0;          // ring index of the current item's first entry
      uint32_t pc[2] = {0u, 0u};  // P tiles consumed per slot
      uint32_t ic[2] = {0u, 0u};  // items per slot
      bool pre = false;           // this item's first scores were issued at the end of the last
      bool ok = true;
      auto wait_entry = [&](uint32_t idx) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(full + idx % kRing, (idx / kRing) & 1u, abort, status));
      };
      // S = Q K^T for slot x into its score columns (query tile b, keys at
      // ring index idx).
      auto issue_qk = [&](int x, uint32_t b, uint32_t idx) {
        const uint32_t tS = tmem + x * 256;
        const uint64_t dq = dq0 + ((b * kTileBytes) >> 4);
        const uint64_t dk = dk0 + (((idx % kRing) * kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tS, dq + kmajor_step(kk, kBM), dk + kmajor_step(kk, kBN), idesc_qk, kk > 0 ? 1u : 0u);
        tc_commit(s_full + x);
      };
      for (int k = 0; ok && seq_valid(k, sh); ++k) {
        const Item it = seq_item(k, sh);
        if (it.n_max == 0) continue;
        for (int i = 0; ok && i <= it.n_max; ++i) {
          const uint32_t ki = base + 2 * i, vi = base + 2 * (i - 1) + 1;
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            const uint32_t tS = tmem + x * 256, tO = tS + 128;
            if (i > 0 && i - 1 < it.n[x]) {
              // O (+)= P_{i-1} V_{i-1}
              if (!(ok = __all_sync(0xffffffffu, mbar_wait(p_ready + x, pc[x] & 1u, abort, status)))) break;
              ++pc[x];
              // The first P.V of an item overwrites O: the epilogue of the
              // slot's previous item must have read it.
              if (i == 1 &&
                  !(ok = __all_sync(0xffffffffu, mbar_wait(tmem_free + x, (ic[x] & 1u) ^ 1u, abort, status))))
                break;
              if ((x == 0 || it.n[0] < i) && !(ok = wait_entry(vi))) break;
              tc_fence_after();
              if (elect_one()) {
                const uint64_t dv = dv0 + (((vi % kRing) * kTileBytes) >> 4);
                // P of keys 0..63 sits in columns 0..31, of keys 64..127 in 64..95.
                mma_ts(tO, tS, dv, idesc_pv, i > 1 ? 1u : 0u);
#pragma unroll
                for (int kk = 1; kk < kBN / 16; ++kk)
                  mma_ts(tO, tS + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8), dv + mnmajor_step(kk), idesc_pv, 1u);
                // Both slots read the tile; release it after the last.
                if (x == 1 || it.n[1] < i) tc_commit(empty + vi % kRing);
              }
            }
            if (i < it.n[x] && !(i == 0 && pre)) {
              // S_i = Q K_i^T
              if (i == 0 && !(ok = __all_sync(0xffffffffu, mbar_wait(q_full + 2 * x + (ic[x] & 1u),
                                                                      (ic[x] >> 1) & 1u, abort, status))))
                break;
              if ((x == 0 || it.n[0] <= i) && !(ok = wait_entry(ki))) break;
              tc_fence_after();
              if (elect_one()) {
                issue_qk(x, 2 * x + (ic[x] & 1u), ki);
                if (x == 1 || it.n[1] <= i) tc_commit(empty + ki % kRing);
              }
            }
          }
          if (!ok) break;
        }
        if (!ok) break;
        // Ring entries: M_{s-1} of this item, then the next item's.
        const uint32_t mi = base + 2 * it.n_max;
        const uint32_t next_base = mi + 1;
        // Retrieval folded into O: O += R' = (rows of sigma(Q), scaled by the
        // softmax warps) M_{s-1}, as soon as a slot's rows are in.  With the
        // gate at exactly 1 the softmax part drops out and R' overwrites O
        // instead.  Then the next item's first scores (a slot's score columns
        // are free once its last P.V, issued before, has read them), so the
        // softmax warps find them ready when they are through with this item.
        const uint64_t dm = dm0 + (((mi % kRing) * kTileBytes) >> 4);
        uint32_t icn[2];
        for (int x = 0; x < 2; ++x) icn[x] = ic[x] + (it.n[x] > 0 ? 1u : 0u);
        Item nx;
        const bool has_next = seq_valid(k + 1, sh);
        if (has_next) nx = seq_item(k + 1, sh);
        const bool next_busy = has_next && nx.n_max > 0;
        bool m_ready = false, k0_ready = false;
        auto retrieval = [&](int x) -> bool {
          const uint32_t icx = x ? ic[1] : ic[0];
          const int hx = x ? it.h[1] : it.h[0];
          const bool keep = gate_sigmoid(__ldg(beta + hx)) != 1.f;
          if (!__all_sync(0xffffffffu, mbar_wait(sq_ready + x, icx & 1u, abort, status))) return false;
          if (!m_ready && !wait_entry(mi)) return false;
          m_ready = true;
          tc_fence_after();
          if (elect_one()) {
            const uint32_t tO = tmem + x * 256 + 128;
            const uint64_t dq = dq0 + (((2 * x + (icx & 1u)) * kTileBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              mma_ss(tO, dq + kmajor_step(kk, kBM), dm + mnmajor_step(kk), idesc_pv, (kk > 0 || keep) ? 1u : 0u);
            tc_commit(r_full + x);
          }
          return true;
        };
        auto first_scores = [&](int x) -> bool {
          const uint32_t icnx = x ? icn[1] : icn[0];
          if (!__all_sync(0xffffffffu, mbar_wait(q_full + 2 * x + (icnx & 1u), (icnx >> 1) & 1u, abort, status)))
            return false;
          if (!k0_ready && !wait_entry(next_base)) return false;
          k0_ready = true;
          tc_fence_after();
          if (elect_one()) issue_qk(x, 2 * x + (icnx & 1u), next_base);
          return true;
        };
        // With equal slots, each slot's next scores go right behind its R';
        // otherwise (the second slot has one key tile less, one query head
        // per KV head) both R' first, which measured faster there.
        const bool interleave = it.n[0] == it.n[1];
        const int nn0 = next_busy ? nx.n[0] : 0, nn1 = next_busy ? nx.n[1] : 0;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          if ((x ? it.n[1] : it.n[0]) > 0 && !(ok = retrieval(x))) break;
          if (interleave && (x ? nn1 : nn0) > 0 && !(ok = first_scores(x))) break;
        }
        if (ok && !interleave) {
#pragma unroll
          for (int x = 0; x < 2; ++x)
            if ((x ? nn1 : nn0) > 0 && !(ok = first_scores(x))) break;
        }
        if (!ok) break;
        if (elect_one()) {
          tc_commit(empty + mi % kRing);
          // Both slots' first scores read K_0 of the next item; release it.
          if (next_busy) tc_commit(empty + next_base % kRing);
        }
        pre = next_busy;
        ic[0] = icn[0];
        ic[1] = icn[1];
        base = next_base;
      }
      // Every MMA issued must be complete before TMEM is released.
      if (elect_one()) tc_commit(drain);
      __syncwarp();
      mbar_wait(drain, 0, abort, status, false);
      __syncwarp();
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // -------------------------------------------------- softmax / epilogue
    // Warpgroup 1 serves slot A, warpgroup 2 slot B: one thread per query row
    // (its TMEM lane).  While one slot's softmax runs, the tensor core works
    // on the other slot.  Waits are made warp-uniform (__all_sync) so that
    // the .sync.aligned TMEM instructions are always executed by full warps.
    const int x = (warp - 4) >> 2;
    const int r = 32 * (warp & 3) + lane;
    const bool leader = (warp & 3) == 0;  // stores the slot's output tiles
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tS = tmem + x * 256 + lane_off;
    const uint32_t tO = tS + 128;
    const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;
    uint32_t sc = 0u, ic = 0u;
    bool store_pending = false;  // (leader, lane 0) a store whose shared-memory reads may still run
    uint32_t pend_b = 0;
    bool ok = true;
    for (int k = 0; ok && seq_valid(k, sh); ++k) {
      const Item it = seq_item(k, sh);
      // (selects, not it.n[x]: a struct indexed by a runtime value would live
      // in local memory, which with almost all of L1 given to shared memory
      // goes to L2)
      const int n = x ? it.n[1] : it.n[0];
      if (n == 0) continue;
      const int qt = x ? it.qt[1] : it.qt[0], h = x ? it.h[1] : it.h[0];
      const uint32_t qb = 2 * x + (ic & 1u);
      unsigned char* sQ = smem + SM::kQ + qb * kTileBytes;
      const float* zs = reinterpret_cast<const float*>(smem + SM::kZ + qb * D * 4);
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < n; ++j) {
        ok = __all_sync(0xffffffffu, mbar_wait(s_full + x, sc & 1u, abort, status));
        ++sc;
        if (!ok) break;
        tc_fence_after();
        uint32_t sv[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sv + c * 32);
        tmem_wait_ld();
        const bool diag = j == qt;
        if (diag) {
          // Diagonal tile: key c is visible to row r iff c <= r.
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c > r) sv[c] = __float_as_uint(-INFINITY);
        }
        // The reference max: the row max of the item's first tile; later
        // tiles are exponentiated against it directly, and only if a row's
        // tile sum exceeds 2^16 (its max grew by more than 2^16 / 128, or
        // overflowed) is the true tile max taken, O and the sum rescaled and
        // the tile redone.  P stays below 2^16 and the reference never falls.
        if (j == 0) m_run = sl2 * row_max128(sv, sv + 64);
        // P (bf16 pairs) over the scores already read: keys 0..63 -> columns
        // 0..31, keys 64..127 -> columns 64..95.
        uint32_t packed[32];
        auto exp_row = [&](float ref) -> float {
          float sum;
          if (diag) {
            sum = exp_pack64<true>(sv, sl2, ref, packed);
            tmem_st32(tS, packed);
            sum += exp_pack64<true>(sv + 64, sl2, ref, packed);
          } else {
            sum = exp_pack64<false>(sv, sl2, ref, packed);
            tmem_st32(tS, packed);
            sum += exp_pack64<false>(sv + 64, sl2, ref, packed);
          }
          tmem_st32(tS + 64, packed);
          return sum;
        };
        float lsum = exp_row(m_run);
        const bool need = !(lsum <= 65536.f);
        if (__any_sync(0xffffffffu, need)) {
          const float mt = need ? sl2 * row_max128(sv, sv + 64) : m_run;
          const float f = need ? ex2_approx(m_run - mt) : 1.f;
#pragma unroll 1
          for (int c = 0; c < D / 16; ++c) {
            uint32_t raw[16];
            tmem_ld16(tO + c * 16, raw);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) raw[e] = __float_as_uint(__uint_as_float(raw[e]) * f);
            tmem_st16(tO + c * 16, raw);
          }
          if (need) {
            l_run *= f;
            m_run = mt;
          }
          // Redo P against the (possibly new) reference (unchanged rows get
          // the same values again).
          lsum = exp_row(m_run);
        }
        l_run += lsum;
        tmem_wait_st();
        tc_fence_before();
        warp_arrive(p_ready + x);
        if (j == 0) {
          // The previous output store of this slot has long read its buffer,
          // which the producer may now refill.
          if (store_pending && lane == 0) {
            tma_store_wait_read();
            mbar_arrive(q_empty + pend_b);
          }
          store_pending = false;
        }
      }
      if (!ok) break;
      // sigma(q_r) and the retrieval denominator sigma(q_r) . z_{s-1} (fp32),
      // in one pass.  (The tile and its z landed before the first scores;
      // the wait makes the copy visible to this thread.  Every QK^T of this
      // slot is complete once its last score tile arrived.)
      ok = __all_sync(0xffffffffu, mbar_wait(q_full + qb, (ic >> 1) & 1u, abort, status));
      if (!ok) break;
      float sg[D];
      const float den = sigma_row<D>(sQ, r, zs, sg);
      // out = (1 - g)/l * O + g/den * sigma(Q) M.  The retrieval enters O
      // through its rows: R' = (sigma(q_r) c_r) M with c_r = g l / ((1 - g) den),
      // so out = (1 - g)/l * (O + R').  With g == 1 (only the retrieval is
      // left) R' overwrites O with c_r = 1/den.  A zero denominator (empty
      // memory) gives a zero retrieval.
      const float gm = gate_sigmoid(__ldg(beta + h));
      float cr, so;
      if (gm == 1.f) {
        cr = den != 0.f ? 1.f / den : 0.f;
        so = 1.f;
      } else {
        cr = den != 0.f ? gm * l_run / ((1.f - gm) * den) : 0.f;
        so = (1.f - gm) / l_run;
      }
      store_scaled_row<D>(sQ, r, sg, cr);
      fence_proxy_async();
      warp_arrive(sq_ready + x);
      ok = __all_sync(0xffffffffu, mbar_wait(r_full + x, ic & 1u, abort, status));
      if (!ok) break;
      tc_fence_after();
      // O read out (then the slot's next P.V may overwrite it), scaled to the
      // output and staged as bf16 in the query tile, whose retrieval rows the
      // tensor core has finished reading; 64 columns per TMEM wait, each
      // chunk straight to the staging tile.
#pragma unroll
      for (int c = 0; c < D; c += 64) {
        uint32_t o_raw[64];
        tmem_ld32(tO + c, o_raw);
        tmem_ld32(tO + c + 32, o_raw + 32);
        tmem_wait_ld();
        uint32_t w[32];
#pragma unroll
        for (int e = 0; e < 32; ++e)
          w[e] = pack_bf16x2(__uint_as_float(o_raw[2 * e]) * so, __uint_as_float(o_raw[2 * e + 1]) * so);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          *reinterpret_cast<uint4*>(sQ + sw128_offset(r, c + e * 8, kBM)) =
              make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
      }
      tc_fence_before();
      warp_arrive(tmem_free + x);
      fence_proxy_async();
      warp_arrive(o_staged + x);
      if (leader) {
        // One TMA store of the tile (rows past the end of the sequence, in a
        // short last segment, are clipped by the tensor bounds).
        ok = __all_sync(0xffffffffu, mbar_wait(o_staged + x, ic & 1u, abort, status));
        if (!ok) break;
        if (lane == 0) {
          for (int p = 0; p < kPanels; ++p)
            tma_store_3d(&tm_o, sQ + p * kBM * 128, p * 64, it.seg0 + qt * kBM, it.b * sh.H_q + h);
          tma_store_commit();
        }
        store_pending = true;
        pend_b = qb;
      }
      ++ic;
    }
    if (leader && lane == 0) tma_store_wait_all();
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

template <int D>
cudaError_t launch(const Problem& p, cudaStream_t stream) {
  CUtensorMap tq, tk, tv, tm, to;
  const uint64_t BHq = (uint64_t)p.B * p.H_q, BHkv = (uint64_t)p.B * p.H_kv;
  if (!make_map(&tq, p.q, D, p.L, BHq, kBM) || !make_map(&tk, p.k, D, p.L, BHkv, kBN) ||
      !make_map(&tv, p.v, D, p.L, BHkv, kBN) || !make_map(&tm, p.M_pref, D, D, (uint64_t)p.T * BHkv, D) ||
      !make_map(&to, p.out, D, p.L, BHq, kBM))
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
  sh.per_group = (sh.g * sh.tps + 1) / 2;  // items per group: pairs of its g * tps query tiles
  sh.upg = (sh.per_group + 1) / 2;
  sh.by_per_group = make_fastdiv((uint32_t)sh.per_group);
  sh.by_upg = make_fastdiv((uint32_t)sh.upg);
  sh.by_H_kv = make_fastdiv((uint32_t)sh.H_kv);
  sh.by_B = make_fastdiv((uint32_t)sh.B);
  const long long units = (long long)p.T * BHkv * sh.upg;
  if ((long long)p.T * BHkv * sh.per_group > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  sh.units = (int)units;
  if (sh.units == 0) return cudaSuccess;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int grid = sh.units < sms ? sh.units : sms;
  const int smem = Smem<D>::kAlloc;
  auto kern = tc_attention<D>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, stream>>>(tq, tk, tv, tm, to, p.z_pref, p.beta, p.status, sh);
  return cudaGetLastError();
}

}  // namespace

bool tc_attention_supported(int d_k, int d_v, int S, bool bf16) {
  return (bf16 && d_k == d_v && (d_k == 64 || d_k == 128) && S % kBM == 0) ||
         tc_small_attention_supported(d_k, d_v, S, bf16);
}

cudaError_t launch_tc_attention(const Problem& p, cudaStream_t stream) {
  // Segments shorter than a query tile: several segments per tile.
  if (p.S < kBM) return launch_tc_small_attention(p, stream);
  // With one query head per KV head a work item pairs query tiles qt and
  // qt - 1 of one head (the second skips the first's last key tile).  At
  // d = 64 the one-tile-per-CTA kernel (two CTAs per SM) is faster there.
  if (p.H_q == p.H_kv && p.d_k == 64) return launch_tc_attention_single(p, stream);
  if (p.d_k == 128) return launch<128>(p, stream);
  if (p.d_k == 64) return launch<64>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace infini
