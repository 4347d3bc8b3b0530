// Memory-state scan for the Infini-attention forward on the tensor-core path
// (sm_100a): segment-parallel products, then a short sequential combine.
//
// The update of one KV head's memory over segment s ("Hugging Face
// Infini-Attention 再現分析", Memory Update; "Leave No Context Behind"
// explainer, "メモリの更新" incl. the delta rule) is affine in M_{s-1}:
//   linear: M_s = M_{s-1} + B_s
//   delta : M_s = M_{s-1} + sigma(K)^T (V - D^-1 sigma(K) M_{s-1})
//               = M_{s-1} - G_s M_{s-1} + B_s
//   with B_s = sigma(K)^T V, G_s = sigma(K)^T D^-1 sigma(K),
//   D = diag(r), r_t = sigma(k_t) . z_{s-1} (rows with r_t = 0 take no
//   retrieval term, i.e. a zero row of D^-1), and z_s = z_{s-1} + sum_t sigma(k_t).
// z does not depend on M, so every segment's (G_s, B_s) can be formed at once:
//   zsum / zprefix (delta only): dz_s = column sums of sigma(K_s), then the
//       prefix z_{s-1} for every segment and z_T;
//   tc_pipe_products (tcgen05, persistent): for every (segment, KV head)
//       item, B_s (and dz_s through a constant ones column, linear rule)
//       and, for the delta rule, G_s = Y^T sigma(K) with Y = D^-1 sigma(K);
//   combine_delta / combine_linear (fp32): walks the segments in order,
//       publishing M_{s-1} (bf16, read by the attention kernel's retrieval)
//       and z_{s-1}, and writes M_T, z_T.
// Precision.  The products' operands are bf16 pairs x = hi + lo
// (hi = bf16(x), lo = bf16(x - hi)), carrying ~16 significant bits:
//   B = hi(sK)^T V + lo(sK)^T V (V is exact in bf16),
//   G = hi(Y)^T hi(sK) + lo(Y)^T hi(sK) + hi(Y)^T lo(sK).
// TMEM accumulates one segment only; the running state is combined in fp32
// on CUDA cores (accumulating a long stream inside the tensor core drifts by
// about one unit in the last place per instruction).
#include <cuda.h>

#include "kernels.h"
#include "packed_math.cuh"
#include "pdl.cuh"
#include "tc_common.cuh"

namespace infini {

namespace {

using namespace tc;

// ---------------------------------------------------------------- dz and z prefix

// Partial column sums of sigma(K): dz[s * C + c][bh][col] = sum over rows t
// of chunk c (of C equal row chunks of segment s) of sigma(k[bh][t][col]).
// Grid (T * C, B*H_kv), block 256 threads: thread (token lane tg, 8-column
// group cg) reads 16-byte pieces of rows tg, tg + NT, ...; the NT partial
// sums of each column are then added in shared memory.  Splitting segments
// into chunks gives the read of K enough CTAs to run at HBM speed.
template <int D>
__global__ void __launch_bounds__(256) zsum(const __nv_bfloat16* __restrict__ k,
                                            float* __restrict__ dz, int L, int S, int C) {
  constexpr int kCG = D / 8;      // 16-byte column groups per row
  constexpr int kNT = 256 / kCG;  // token lanes
  __shared__ float part[kNT * D];
  pdl_trigger();
  pdl_wait();
  const int s = blockIdx.x / C, c = blockIdx.x % C, bh = blockIdx.y, tid = threadIdx.x;
  const int cg = tid % kCG, tg = tid / kCG;
  const int chunk = (S + C - 1) / C;
  const int r0 = s * S + c * chunk, r1 = min(min(r0 + chunk, s * S + S), L);
  const uint4* base = reinterpret_cast<const uint4*>(k + (size_t)bh * L * D) + cg;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll 4
  for (int t = r0 + tg; t < r1; t += kNT) {
    const uint4 v = __ldg(base + (size_t)t * kCG);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] += elu1_fast(__uint_as_float(w[i] << 16));
      acc[2 * i + 1] += elu1_fast(__uint_as_float(w[i] & 0xFFFF0000u));
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) part[tg * D + cg * 8 + i] = acc[i];
  __syncthreads();
  if (tid < D) {
    float sum = 0.f;
#pragma unroll 8
    for (int j = 0; j < kNT; ++j) sum += part[j * D + tid];
    dz[((size_t)blockIdx.x * gridDim.y + bh) * D + tid] = sum;
  }
}

// z_{s-1} for s = 0..T-1 into z_pref (slot 0 = z_in) and z_T, from the C
// chunk partials of every segment.  Grid (B*H_kv), block 1024 threads: column
// c of z and a group g of kSG = 1024 / D contiguous segment ranges per
// thread.  Each group sums its range (the partials loaded kAhead at a time,
// so that a range costs about one memory round trip), the groups' totals are
// added in group order through shared memory, and each group then walks its
// range again from that offset, writing z_{s-1} at every segment start.
template <int D>
__global__ void __launch_bounds__(1024) zprefix(const float* __restrict__ dz, const float* z_in,
                                                float* __restrict__ z_pref, float* z_out, int T,
                                                int C) {
  constexpr int kSG = 1024 / D;
  constexpr int kAhead = 16;
  __shared__ float tot[kSG][D];
  pdl_trigger();
  pdl_wait();
  const int bh = blockIdx.x, c = threadIdx.x % D, g = threadIdx.x / D, BH = gridDim.x;
  const int per = (T + kSG - 1) / kSG;
  const int s0 = min(T, g * per), s1 = min(T, s0 + per);
  const int i0 = s0 * C, i1 = s1 * C;
  auto part_at = [&](int i) { return dz[((size_t)i * BH + bh) * D + c]; };
  // (z_out may be z_in: every thread reads its entry before the barrier, and
  // only the last group writes z_out, after it)
  const float zin = z_in[(size_t)bh * D + c];
  // The range's total, segment by segment in order.
  float total = 0.f, seg = 0.f;
  for (int b0 = i0; b0 < i1; b0 += kAhead) {
    float part[kAhead];
#pragma unroll
    for (int u = 0; u < kAhead; ++u) part[u] = b0 + u < i1 ? part_at(b0 + u) : 0.f;
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
      const int i = b0 + u;
      if (i >= i1) break;
      seg += part[u];
      if (i % C == C - 1) {
        total += seg;
        seg = 0.f;
      }
    }
  }
  tot[g][c] = total;
  __syncthreads();
  float z = zin;
  for (int h = 0; h < g; ++h) z += tot[h][c];
  // The walk over the range from its offset.
  seg = 0.f;
  for (int b0 = i0; b0 < i1; b0 += kAhead) {
    float part[kAhead];
#pragma unroll
    for (int u = 0; u < kAhead; ++u) part[u] = b0 + u < i1 ? part_at(b0 + u) : 0.f;
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
      const int i = b0 + u;
      if (i >= i1) break;
      const int j = i % C;
      if (j == 0) z_pref[((size_t)(i / C) * BH + bh) * D + c] = z;
      seg += part[u];
      if (j == C - 1) {
        z += seg;
        seg = 0.f;
      }
    }
  }
  if (g == kSG - 1) z_out[(size_t)bh * D + c] = z;
}

constexpr int kZChunksMax = 8;

// Row chunks per segment for zsum: about 256 rows each, at most kZChunksMax.
int zsum_chunks(int S) { return S >= 256 * kZChunksMax ? kZChunksMax : (S >= 512 ? S / 256 : 1); }

// ---------------------------------------------------------------- pipelined products

// Per (segment, KV head), streamed in 64-token blocks:
//   linear: B_s = sigma(K_s)^T V_s and dz_s = column sums of sigma(K_s);
//   delta : B_s as above and G_s = Y^T sigma(K_s), Y = D^-1 sigma(K_s),
//           D = diag(sigma(K_s) z_{s-1}) (rows with r_t = 0 give zero rows).
// A TMA ring of (K, V) blocks; sigma(K) (and Y) as bf16 hi/lo pairs in two
// alternating operand buffers, so the math warps build block b+1 while the
// tensor core multiplies block b; dz (linear) by the tensor core too, from
// a constant operand whose first column is ones.
// Persistent: one CTA per SM walks the (segment, KV head) items, with the
// block counters running on across items, so the producer streams the next
// items' blocks ahead.  Two TMEM accumulators alternate between items (an
// accumulator goes back to the MMA warp through its acc_empty barrier); for
// d = 64, whose items can be a single block, the math warps write item j's
// products out of TMEM only after building the first block of item j + 1,
// so that the tensor core works meanwhile.  (For d = 128 the epilogue
// follows the item's last block: items are long there, and the 576-thread
// CTA has no registers to spare inside the block loop.)
// The linear rule is HBM-bound (each block brings 2 x 64 x d bf16 of K and
// V); the delta rule does 20 MMAs (128 x d x 16) per block.  For d = 64 the
// products' M = 128 operands (sigma(K)^T, Y^T) carry a zero upper half.
constexpr int kLTok = 64;      // tokens per block

template <int D_, bool DELTA>
struct PipeSmem {
  static constexpr int kD = D_;
  // Math warps: 2 tokens per thread and block, 8 columns per thread (16
  // warps for d = 128, 8 for d = 64), to hide the latency of the sigma
  // chain -- and, for the delta rule, of r_t's shuffle sum and 1/r_t; the
  // parts go straight to the operand buffer.
  static constexpr int kMath = kD / 8;
  static constexpr int kThreads = 64 + 32 * kMath;
  static constexpr int kCG = kD / 8;                      // 8-column chunks per token
  static constexpr int kTL = 32 * kMath / kCG;            // token lanes
  static constexpr int kTokPerThread = kLTok / kTL;
  static constexpr int kStages = DELTA ? 256 / kD : 512 / kD;  // K/V ring depth
  static constexpr int kPanel = kLTok * 128;              // 64 rows x 128 B
  static constexpr int kBlk = kLTok * kD * 2;             // one 64 x d bf16 block
  static constexpr int kStage = 2 * kBlk;                 // K then V
  static constexpr int kHalf = kLTok * 128 * 2;           // one 64 x 128 operand part
  static constexpr int kOpParts = DELTA ? 4 : 2;          // sigma hi, lo (, Y hi, lo)
  static constexpr int kRing = 0;
  static constexpr int kOp = kRing + kStages * kStage;    // [2][parts]
  // Linear rule: a constant [64 tokens][64] panel whose column 0 is 1.0, the
  // B operand of the MMA that sums sigma(K) over the tokens (dz).
  static constexpr int kOnes = kOp + 2 * kOpParts * kHalf;
  static constexpr int kBar = kOnes + (DELTA ? 0 : kPanel);
  // full[kStages] empty[kStages] op_full[2] op_empty[2] acc_full[2] acc_empty[2] drain
  static constexpr int kNumBars = 2 * kStages + 9;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kAlloc = kAbort + 4 + 1024;
  // TMEM: two accumulators of 256 columns, delta [G | B], linear [B | dz
  // (16 columns, column 0 used)].
  static constexpr uint32_t kAccCols = 256;
  static constexpr uint32_t kTmemCols = 2 * kAccCols;
  static_assert(kOnes % 1024 == 0 && kTokPerThread * kTL == kLTok, "pipe layout");
};

template <int D_, bool DELTA>
__global__ void __launch_bounds__(PipeSmem<D_, DELTA>::kThreads, 1)
tc_pipe_products(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                 const float* __restrict__ z_pref, float* __restrict__ Gbuf, float* __restrict__ Bbuf,
                 float* __restrict__ dz, unsigned int* __restrict__ status, int L, int S, int T,
                 int BH) {
  using SM = PipeSmem<D_, DELTA>;
  constexpr int D = SM::kD;
  constexpr int kStages = SM::kStages;
  constexpr int kLMath = SM::kMath;
  constexpr int kTL = SM::kTL;
  constexpr int kTPT = SM::kTokPerThread;
  const int items = T * BH;
  // Item -> (segment s = item % T, KV head bh = item / T).
  auto item_blocks = [&](int item) {
    const int seg_len = min(S, L - (item % T) * S);
    return (seg_len + kLTok - 1) / kLTok;
  };

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* ring = smem + SM::kRing;
  unsigned char* op = smem + SM::kOp;
  unsigned char* ones = smem + SM::kOnes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* op_full = bars + 2 * kStages;
  uint64_t* op_empty = op_full + 2;
  uint64_t* acc_full = op_empty + 2;    // [2]
  uint64_t* acc_empty = acc_full + 2;   // [2]
  uint64_t* drain = acc_empty + 2;
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
    for (int i = 0; i < kStages; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, kLMath + 1);  // math warps (K read) + the MMA commit (V read)
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(op_full + i, kLMath);
      mbar_init(op_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full + i, 1);
      mbar_init(acc_empty + i, kLMath);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (D < 128) {
    // The operand parts' upper panel (rows D..127 of sigma(K)^T, Y^T) stays 0.
    for (int i = threadIdx.x; i < 2 * SM::kOpParts * SM::kHalf / 16; i += SM::kThreads)
      *reinterpret_cast<uint4*>(op + i * 16) = make_uint4(0, 0, 0, 0);
  }
  if (!DELTA) {
    // Row t of the ones panel: its 16-byte chunk that holds logical column 0
    // sits at chunk (t & 7) under the 128-byte swizzle.
    for (int i = threadIdx.x; i < kLTok * 8; i += SM::kThreads) {
      const int row = i / 8, chunk = i % 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (chunk == (row & 7)) v.x = 0x3F80u;  // element (row, 0) = bf16(1.0)
      *reinterpret_cast<uint4*>(ones + i * 16) = v;
    }
  }
  fence_proxy_async();
  if (warp == 1) {
    tmem_alloc(tmem_slot, SM::kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();
  pdl_wait();  // (nothing above touched global memory)
  // Accumulator a: G at 0 and B at 128 (delta), B at 0 and dz at 128 (linear).
  auto tG = [&](int a) { return tmem + a * SM::kAccCols; };
  auto tB = [&](int a) { return tmem + a * SM::kAccCols + (DELTA ? 128 : 0); };
  // d = 64, linear rule: V's panel and the ones panel form one N = 80 operand
  // (the descriptor's panel stride reaches from the ring stage to the ones
  // panel), so dz lands in columns 64.. of the B accumulator with no MMAs of
  // its own; d = 128 keeps the separate N = 16 dz MMAs (its three panels
  // would need one stride).
  constexpr bool kFusedDz = !DELTA && D_ == 64;
  auto tDZ = [&](int a) { return tmem + a * SM::kAccCols + (kFusedDz ? 64 : 128); };

  if (warp == 0) {
    // ---------------------------------------------- TMA producer (whole warp waits, one elected lane issues)
    int gb = 0;  // blocks issued so far (all items)
    bool ok = true;
    for (int item = blockIdx.x; ok && item < items; item += gridDim.x) {
      const int seg0 = (item % T) * S, bh = item / T, nblk = item_blocks(item);
      for (int b = 0; b < nblk; ++b, ++gb) {
        const int st = gb % kStages;
        const uint32_t ph = (uint32_t)(gb / kStages) & 1u;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(empty + st, ph ^ 1u, abort, status)))) break;
        if (elect_one()) {
          unsigned char* dst = ring + st * SM::kStage;
          mbar_arrive_expect_tx(full + st, SM::kStage);
          for (int p = 0; p < D / 64; ++p) {
            tma_load_3d(dst + p * SM::kPanel, &tm_k, full + st, p * 64, seg0 + b * kLTok, bh);
            tma_load_3d(dst + SM::kBlk + p * SM::kPanel, &tm_v, full + st, p * 64, seg0 + b * kLTok, bh);
          }
        }
      }
    }
    // Every copy issued must land before the CTA exits.
    for (int b = max(0, gb - kStages); b < gb; ++b)
      mbar_wait(full + b % kStages, (uint32_t)(b / kStages) & 1u, abort, status, false);
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------- MMA issuer (whole warp waits, one elected lane issues)
    constexpr uint32_t idesc = idesc_bf16_f32(128, D, true, true);
    constexpr uint32_t idesc_dz = idesc_bf16_f32(128, 16, true, true);
    constexpr uint32_t idesc_vz = idesc_bf16_f32(128, D + 16, true, true);  // [V | ones]
    const uint64_t dop = sw128_desc(smem_u32(op), SM::kPanel, 1024);
    const uint64_t dring = sw128_desc(smem_u32(ring + SM::kBlk), SM::kPanel, 1024);
    const uint64_t dones = sw128_desc(smem_u32(ones), SM::kPanel, 1024);
    bool ok = true;
    int gb = 0, j = 0;  // blocks and items so far
    for (int item = blockIdx.x; ok && item < items; item += gridDim.x, ++j) {
      const int nblk = item_blocks(item), a = j & 1;
      // Accumulator a is free once the math warps have read item j - 2's.
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(acc_empty + a, ((uint32_t)(j >> 1) & 1u) ^ 1u, abort, status)))) break;
      for (int b = 0; b < nblk; ++b, ++gb) {
        const int st = gb % kStages, ob = gb & 1;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(op_full + ob, (uint32_t)(gb >> 1) & 1u, abort, status)))) break;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(full + st, (uint32_t)(gb / kStages) & 1u, abort, status)))) break;
        tc_fence_after();
        if (elect_one()) {
          // Operand parts: sigma hi, sigma lo, (Y hi, Y lo).
          const uint64_t shi = dop + ((ob * SM::kOpParts * SM::kHalf) >> 4);
          const uint64_t slo = shi + (SM::kHalf >> 4);
          const uint64_t yhi = shi + ((2 * SM::kHalf) >> 4);
          const uint64_t ylo = shi + ((3 * SM::kHalf) >> 4);
          const uint64_t vv = dring + ((st * SM::kStage) >> 4);
          // [V | ones]: V's panel, then the ones panel as the second one.
          const uint32_t v_off = SM::kRing + st * SM::kStage + SM::kBlk;
          const uint64_t vz = sw128_desc(smem_u32(ring + st * SM::kStage + SM::kBlk),
                                         (uint32_t)SM::kOnes - v_off, 1024);
#pragma unroll
          for (int kk = 0; kk < kLTok / 16; ++kk) {
            const uint32_t stp = mnmajor_step(kk);
            const uint32_t acc = (b > 0 || kk > 0) ? 1u : 0u;
            if (DELTA) {
              mma_ss(tG(a), yhi + stp, shi + stp, idesc, acc);
              mma_ss(tG(a), ylo + stp, shi + stp, idesc, 1u);
              mma_ss(tG(a), yhi + stp, slo + stp, idesc, 1u);
            }
            if (kFusedDz) {
              mma_ss(tB(a), shi + stp, vz + stp, idesc_vz, acc);
              mma_ss(tB(a), slo + stp, vz + stp, idesc_vz, 1u);
            } else {
              mma_ss(tB(a), shi + stp, vv + stp, idesc, acc);
              mma_ss(tB(a), slo + stp, vv + stp, idesc, 1u);
            }
            if (!DELTA && !kFusedDz) {
              mma_ss(tDZ(a), shi + stp, dones + stp, idesc_dz, acc);
              mma_ss(tDZ(a), slo + stp, dones + stp, idesc_dz, 1u);
            }
          }
          tc_commit(op_empty + ob);
          tc_commit(empty + st);
          if (b == nblk - 1) tc_commit(acc_full + a);
        }
      }
    }
    // Every MMA issued must complete before the accumulator is released.
    if (elect_one()) tc_commit(drain);
    __syncwarp();
    mbar_wait(drain, 0, abort, status, false);
    __syncwarp();
  } else {
    // ---------------------------------------------- math warps
    // Thread (column chunk cg of 8 columns, token lane tl): tokens tl,
    // tl + kTL, ...; the D/8 threads of a token are consecutive lanes of one
    // warp.  Epilogue: TMEM lane k = row k of the products.
    const int mt = threadIdx.x - 64;
    const int cg = mt % SM::kCG, tl = mt / SM::kCG;
    const int k = 32 * (warp & 3) + lane, quarter = (warp - 2) >> 2;  // 0..kMath/4-1
    const uint32_t lq = (uint32_t)(32 * (warp & 3)) << 16;
    // Item jj's products (slice sl) out of accumulator jj & 1: kMath / 4
    // warps per TMEM lane quarter share the row's columns, delta [G | B]
    // (2D columns), linear B (D columns) and dz.  For D = 64 only lanes
    // 0..63 hold rows.
    auto epilogue = [&](int jj, size_t sl) -> bool {
      const int a = jj & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(acc_full + a, (uint32_t)(jj >> 1) & 1u, abort, status)))
        return false;
      tc_fence_after();
      constexpr int kParts = kLMath / 4;
      constexpr int kCols = (DELTA ? 2 * D : D) / kParts;  // columns per warp
      if (k < D) {
        if (!DELTA && quarter == 0) {
          // dz_k: column 0 of the ones-column accumulator.
          uint32_t v[32];
          tmem_ld32(tDZ(a) + lq, v);
          tmem_wait_ld();
          dz[sl * D + k] = __uint_as_float(v[0]);
        }
#pragma unroll
        for (int c = 0; c < kCols / 32; ++c) {
          const int col = kCols * quarter + 32 * c;  // of [G | B] or of B
          const bool isB = !DELTA || col >= D;
          const int cc = DELTA && col >= D ? col - D : col;
          uint32_t v[32];
          tmem_ld32((isB ? tB(a) : tG(a)) + lq + cc, v);
          tmem_wait_ld();
          float4* dst = reinterpret_cast<float4*>((isB ? Bbuf : Gbuf) + (sl * D + k) * D + cc);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                 __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty + a);
      return true;
    };
    auto load_z = [&](int item, float* zc) {
      const size_t sl = (size_t)(item % T) * BH + item / T;
      const float4 za = *reinterpret_cast<const float4*>(z_pref + sl * D + 8 * cg);
      const float4 zb = *reinterpret_cast<const float4*>(z_pref + sl * D + 8 * cg + 4);
      zc[0] = za.x; zc[1] = za.y; zc[2] = za.z; zc[3] = za.w;
      zc[4] = zb.x; zc[5] = zb.y; zc[6] = zb.z; zc[7] = zb.w;
    };
    bool ok = true;
    int gb = 0, j = 0;
    size_t prev_slice = 0;  // item j - 1's slice, whose products are still in TMEM
    // d = 64 (short items, registers to spare) writes item j's products
    // after item j + 1's first block, and loads z_{s-1} one item ahead.
    constexpr bool kLag = D < 128, kZAhead = D < 128;
    float zc[8], zn[8];
    if (DELTA && kZAhead && blockIdx.x < items) load_z(blockIdx.x, zn);
    for (int item = blockIdx.x; ok && item < items; item += gridDim.x, ++j) {
      const int s = item % T, bh = item / T, nblk = item_blocks(item);
      const int seg_len = min(S, L - s * S);
      const size_t slice = (size_t)s * BH + bh;
      if (DELTA && kZAhead) {
        // z_{s-1} of this item (loaded one item ahead), then the next item's.
#pragma unroll
        for (int i = 0; i < 8; ++i) zc[i] = zn[i];
        if (item + (int)gridDim.x < items) load_z(item + gridDim.x, zn);
      } else if (DELTA) {
        load_z(item, zc);
      }
      for (int b = 0; b < nblk; ++b, ++gb) {
        const int st = gb % kStages, ob = gb & 1;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(full + st, (uint32_t)(gb / kStages) & 1u, abort, status)))) break;
        const unsigned char* kb = ring + st * SM::kStage;
        // The operand buffer is free once the MMAs of block gb - 2 are done
        // (long before, normally); the parts go straight into it.
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(op_empty + ob, ((uint32_t)(gb >> 1) & 1u) ^ 1u, abort, status)))) break;
        unsigned char* hb = op + ob * SM::kOpParts * SM::kHalf;
#pragma unroll
        for (int i = 0; i < kTPT; ++i) {
          const int t = tl + kTL * i;
          const bool valid = b * kLTok + t < seg_len;
          const uint32_t off = sw128_offset(t, 8 * cg, kLTok);
          uint4 kv = *reinterpret_cast<const uint4*>(kb + off);
          // (rows past the segment: sigma = 0 exactly)
          if (!valid) kv = make_uint4(0xFF7FFF7Fu, 0xFF7FFF7Fu, 0xFF7FFF7Fu, 0xFF7FFF7Fu);
          const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
          float2 sg[4];
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            sg[e] = pk::sigma_pair(kw[e]);
            pk::split_pair(sg[e], hw[e], lw[e]);
          }
          *reinterpret_cast<uint4*>(hb + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(hb + SM::kHalf + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
          if (DELTA) {
            // r_t = sigma(k_t) . z_{s-1} over the token's D/8 threads; Y = sigma / r.
            float r = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              r = fmaf(sg[e].x, zc[2 * e], r);
              r = fmaf(sg[e].y, zc[2 * e + 1], r);
            }
#pragma unroll
            for (int o = SM::kCG / 2; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
            const float w = r != 0.f ? 1.f / r : 0.f;
            uint32_t yh[4], yl[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) pk::split_pair(pk::mul2(make_float2(w, w), sg[e]), yh[e], yl[e]);
            *reinterpret_cast<uint4*>(hb + 2 * SM::kHalf + off) = make_uint4(yh[0], yh[1], yh[2], yh[3]);
            *reinterpret_cast<uint4*>(hb + 3 * SM::kHalf + off) = make_uint4(yl[0], yl[1], yl[2], yl[3]);
          }
        }
        // K of this block has been read.
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + st);
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(op_full + ob);
        // With the tensor core fed, the previous item's products.
        if (kLag && b == 0 && j > 0 && !(ok = epilogue(j - 1, prev_slice))) break;
      }
      if (!kLag && ok) ok = epilogue(j, slice);
      prev_slice = slice;
    }
    if (kLag && ok && j > 0) ok = epilogue(j - 1, prev_slice);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, SM::kTmemCols);
  }
}

// ---------------------------------------------------------------- sequential combine

constexpr int kCB = 16;  // columns of M per combine CTA (delta)

// Four consecutive elements of a published state M_{s-1}: bf16 for the
// attention's retrieval, or fp32 (the backward's recompute of the states).
__device__ __forceinline__ void store_state4(__nv_bfloat16* dst, float4 m) {
  uint2 w;
  w.x = pack_bf16x2(m.x, m.y);
  w.y = pack_bf16x2(m.z, m.w);
  *reinterpret_cast<uint2*>(dst) = w;
}
__device__ __forceinline__ void store_state4(float* dst, float4 m) {
  *reinterpret_cast<float4*>(dst) = m;
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Delta rule: M_s = M_{s-1} - G_s M_{s-1} + B_s on columns [16 cb, 16 cb + 16).
// Grid (B*H_kv, D/16), block D threads (D/32 warps).  Thread tile: 4 rows x
// 4 columns of M, lane -> (row group lane / 4 of the warp's 32 rows, column
// group lane % 4), so that one 128-bit shared load of G and one of M_{s-1}
// per kk feed 16 FMAs (8 fma.rn.f32x2), and a warp's loads per kk are two
// shared-memory wavefronts: the loop is bound by the FMA pipe, not by
// shared-memory bandwidth.  G_s is symmetric up to the rounding of its bf16
// pair products (the dropped lo*lo term, ~2^-16 relative), so row k of
// G_s M is read from column k of G_s: four consecutive rows of the tile are
// one contiguous 16-byte piece.  G_{s+1} streams in (cp.async) and the B_{s+2}
// tile is loaded into registers while step s runs (one step ahead left the
// load's latency exposed: 40.6 -> 36.8 us at the 200M shape, 54 -> 47 us at
// 8B).  Plain block barriers only.
template <int D, typename MP>
__global__ void __launch_bounds__(D) combine_delta(const float* __restrict__ M_in,
                                                   const float* __restrict__ Gbuf,
                                                   const float* __restrict__ Bbuf,
                                                   MP* __restrict__ M_pref,
                                                   float* __restrict__ M_out, int T) {
  static_assert(kCB == 16 && D % 32 == 0, "combine_delta thread map");
  extern __shared__ __align__(16) float csm[];
  // (The successor may launch only once the walk is done: CTAs parked in
  // pdl_wait beside this latency-bound walk were measured to slow it.)
  pdl_wait();
  float* sG = csm;               // two G_s buffers [D][D]
  float* sM = csm + 2 * D * D;   // M_{s-1}[:, 16 columns]
  const int bh = blockIdx.x, c0 = blockIdx.y * kCB, BH = gridDim.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int k0 = 32 * warp + 4 * (lane >> 2);  // first of the tile's 4 rows
  const int c = 4 * (lane & 3);                // first of its 4 columns (in the CTA's 16)
  auto load_g = [&](int s, float* dst) {
    const float4* src = reinterpret_cast<const float4*>(Gbuf + ((size_t)s * BH + bh) * D * D);
    for (int e = tid; e < D * D / 4; e += D) cp_async16(dst + 4 * e, src + e);
    cp_async_commit();
  };
  auto load_b = [&](int s, float4* dst) {
    const float* src = Bbuf + (((size_t)s * BH + bh) * D + k0) * D + c0 + c;
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = *reinterpret_cast<const float4*>(src + (size_t)i * D);
  };
  float4 m[4];  // M[k0 + i][c0 + c .. + 3]
#pragma unroll
  for (int i = 0; i < 4; ++i)
    m[i] = *reinterpret_cast<const float4*>(M_in + ((size_t)bh * D + k0 + i) * D + c0 + c);
  // B_s, B_{s+1} in registers; B_{s+2} is loaded during step s (a step is
  // shorter than a load's latency).
  float4 bq[4], bn[4];
  load_g(0, sG);
  load_b(0, bq);
  if (T > 1) load_b(1, bn);
  for (int s = 0; s < T; ++s) {
    const size_t slice = (size_t)s * BH + bh;
    float4 bn2[4] = {};
    if (s + 2 < T) load_b(s + 2, bn2);
    float* G = sG + (s & 1) * D * D;
    if (s + 1 < T) {
      load_g(s + 1, sG + ((s + 1) & 1) * D * D);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    // Publish M_{s-1} for segment s's retrieval.
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      store_state4(M_pref + (slice * D + k0 + i) * D + c0 + c, m[i]);
      *reinterpret_cast<float4*>(sM + (k0 + i) * kCB + c) = m[i];
    }
    __syncthreads();
    // (G_s M)[k0 + i][c .. c + 3] as column pairs.
    float2 acc[4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = make_float2(0.f, 0.f);
#pragma unroll 4
    for (int kk = 0; kk < D; ++kk) {
      const float4 g = *reinterpret_cast<const float4*>(G + kk * D + k0);
      const float4 mv = *reinterpret_cast<const float4*>(sM + kk * kCB + c);
      const float2 mlo = make_float2(mv.x, mv.y), mhi = make_float2(mv.z, mv.w);
      const float gr[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 g2 = make_float2(gr[i], gr[i]);
        acc[i][0] = pk::fma2(g2, mlo, acc[i][0]);
        acc[i][1] = pk::fma2(g2, mhi, acc[i][1]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      m[i].x = (m[i].x - acc[i][0].x) + bq[i].x;
      m[i].y = (m[i].y - acc[i][0].y) + bq[i].y;
      m[i].z = (m[i].z - acc[i][1].x) + bq[i].z;
      m[i].w = (m[i].w - acc[i][1].y) + bq[i].w;
      bq[i] = bn[i];
      bn[i] = bn2[i];
    }
    __syncthreads();
  }
  pdl_trigger();
#pragma unroll
  for (int i = 0; i < 4; ++i)
    *reinterpret_cast<float4*>(M_out + ((size_t)bh * D + k0 + i) * D + c0 + c) = m[i];
}

// Linear rule: M_s = M_{s-1} + B_s, z_s = z_{s-1} + dz_s, element-parallel.
// Grid (B*H_kv, ceil(D*D / 1024)), block 256 threads x 4 elements; block
// (bh, 0) also carries z.
template <int D, typename MP>
__global__ void __launch_bounds__(256) combine_linear(const float* __restrict__ M_in,
                                                      const float* __restrict__ Bbuf,
                                                      const float* __restrict__ dz,
                                                      MP* __restrict__ M_pref,
                                                      const float* z_in,
                                                      float* __restrict__ z_pref,
                                                      float* __restrict__ M_out, float* z_out,
                                                      int T) {
  pdl_trigger();
  pdl_wait();
  const int bh = blockIdx.x, BH = gridDim.x;
  const int e = (blockIdx.y * 256 + threadIdx.x) * 4;  // element of the D x D matrix
  if (e < D * D) {
    float4 m = *reinterpret_cast<const float4*>(M_in + (size_t)bh * D * D + e);
    // The products of kAhead segments are loaded before they are added, so
    // that many loads are in flight per thread (the walk itself is serial).
    constexpr int kAhead = 8;
    for (int s0 = 0; s0 < T; s0 += kAhead) {
      float4 b[kAhead];
#pragma unroll
      for (int i = 0; i < kAhead; ++i)
        if (s0 + i < T)
          b[i] = *reinterpret_cast<const float4*>(Bbuf + ((size_t)(s0 + i) * BH + bh) * D * D + e);
#pragma unroll
      for (int i = 0; i < kAhead; ++i) {
        if (s0 + i >= T) break;
        store_state4(M_pref + ((size_t)(s0 + i) * BH + bh) * D * D + e, m);
        m.x += b[i].x;
        m.y += b[i].y;
        m.z += b[i].z;
        m.w += b[i].w;
      }
    }
    *reinterpret_cast<float4*>(M_out + (size_t)bh * D * D + e) = m;
  }
  if (blockIdx.y == 0 && threadIdx.x < D) {
    const int c = threadIdx.x;
    // (z_out may be z_in: this thread reads its entry before it writes it)
    float z = z_in[(size_t)bh * D + c];
    z_pref[(size_t)bh * D + c] = z;  // slot 0, read by segment 0
    for (int s = 1; s < T; ++s) {
      z += dz[((size_t)(s - 1) * BH + bh) * D + c];
      z_pref[((size_t)s * BH + bh) * D + c] = z;
    }
    z_out[(size_t)bh * D + c] = z + dz[((size_t)(T - 1) * BH + bh) * D + c];
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

template <int D, bool DELTA>
cudaError_t launch_pipe_products(const Problem& p, cudaStream_t stream) {
  CUtensorMap lk, lv;
  const uint64_t BHkv = (uint64_t)p.B * p.H_kv;
  if (!make_map(&lk, p.k, D, p.L, BHkv, kLTok) || !make_map(&lv, p.v, D, p.L, BHkv, kLTok))
    return cudaErrorInvalidValue;
  const int smem = PipeSmem<D, DELTA>::kAlloc;
  auto kern = tc_pipe_products<D, DELTA>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const long items = (long)p.T * (long)BHkv;
  const int grid = (int)(items < sms ? items : sms);  // persistent: one CTA per SM
  return launch_pdl(!DELTA, kern, dim3(grid), dim3(PipeSmem<D, DELTA>::kThreads), smem, stream, lk, lv,
                    (const float*)p.z_pref, p.Gbuf, p.Bbuf, p.dz, p.status, p.L, p.S, p.T, (int)BHkv);
}

// Launch chain.  The linear rule's kernels (products, combine) and the
// attention after them are launched with programmatic dependent launch: the
// next kernel's launch and prologue overlap the previous one's tail (200M
// shape: 56 -> 52 us per forward).  The delta rule's chain is launched
// plainly: with every link dependent, the forward took 129 us against 116.
template <int D, typename MP>
cudaError_t launch(const Problem& p, cudaStream_t stream) {
  const unsigned BH = (unsigned)((uint64_t)p.B * p.H_kv);
  MP* Mp = static_cast<MP*>(p.M_pref);
  cudaError_t e;
  if (p.delta) {
    const int C = zsum_chunks(p.S);
    if ((e = launch_pdl(false, zsum<D>, dim3(p.T * C, BH), dim3(256), 0, stream,
                        static_cast<const __nv_bfloat16*>(p.k), p.dz, p.L, p.S, C)) != cudaSuccess)
      return e;
    if ((e = launch_pdl(false, zprefix<D>, dim3(BH), dim3(1024), 0, stream, (const float*)p.dz, p.z_in, p.z_pref,
                        p.z_out, p.T, C)) != cudaSuccess)
      return e;
    e = launch_pipe_products<D, true>(p, stream);
    if (e != cudaSuccess) return e;
    const int csmem = (2 * D * D + D * kCB) * (int)sizeof(float);
    e = cudaFuncSetAttribute(combine_delta<D, MP>, cudaFuncAttributeMaxDynamicSharedMemorySize, csmem);
    if (e != cudaSuccess) return e;
    return launch_pdl(false, combine_delta<D, MP>, dim3(BH, D / kCB), dim3(D), csmem, stream, p.M_in,
                      (const float*)p.Gbuf, (const float*)p.Bbuf, Mp, p.M_out, p.T);
  }
  e = launch_pipe_products<D, false>(p, stream);
  if (e != cudaSuccess) return e;
  return launch_pdl(true, combine_linear<D, MP>, dim3(BH, (D * D + 1023) / 1024), dim3(256), 0, stream,
                    p.M_in, (const float*)p.Bbuf, (const float*)p.dz, Mp, p.z_in, p.z_pref, p.M_out,
                    p.z_out, p.T);
}

}  // namespace

bool tc_scan_supported(int d_k, int d_v, bool bf16) {
  return bf16 && d_k == d_v && (d_k == 64 || d_k == 128);
}

int tc_scan_launches(bool delta) { return delta ? 4 : 2; }

void tc_scan_workspace(int B, int H_kv, int T, int d, bool delta, size_t* g_bytes, size_t* b_bytes,
                       size_t* dz_bytes) {
  const size_t slices = (size_t)T * B * H_kv;
  *g_bytes = delta ? slices * d * d * 4 : 0;
  *b_bytes = slices * d * d * 4;
  // The delta rule's column sums come in up to kZChunksMax chunk partials.
  *dz_bytes = slices * d * 4 * (delta ? kZChunksMax : 1);
}

cudaError_t launch_tc_state_scan(const Problem& p, cudaStream_t stream) {
  if (p.M_pref_bf16) {
    if (p.d_k == 128) return launch<128, __nv_bfloat16>(p, stream);
    if (p.d_k == 64) return launch<64, __nv_bfloat16>(p, stream);
  } else {
    if (p.d_k == 128) return launch<128, float>(p, stream);
    if (p.d_k == 64) return launch<64, float>(p, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace infini
