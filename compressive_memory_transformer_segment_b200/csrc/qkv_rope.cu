// Q/K/V projections with rotary position embedding: the prologue that turns
// a layer's input into the query, key and value heads that the segment
// attention and the compressive memory share ("Leave No Context Behind"
// explainer, "メモリ構造": the memory reuses the attention's Q/K/V; "Как
// работает Infini-attention", section 9: linear Q/K/V layers over the input).
//
//   y = x W^T (+ bias)     x [rows = B*L, d_model], W [N = (H_q + 2 H_kv) d, d_model]
//   query and key heads rotated token by token (rotate-half pairing: element
//   i with element i + d/2, by the angle whose cos / sin sit in row t of the
//   tables), values not;
//   written in bf16 as q [B, H_q, L, d], k and v [B, H_kv, L, d].
//
// qkv_rope (tcgen05, persistent): one CTA per SM walks 128 x 256 output tiles
// in row-tile-major order, so the CTAs in flight share each 128-row slab of x
// and all of W through L2.  A 4-stage TMA ring of 64-wide K slices (x 16 KB +
// W 32 KB, 128-byte swizzle); one elected thread issues four 128 x 256 x 16
// MMAs per slice into one of two TMEM accumulators (256 columns each); four
// epilogue warps (thread = output row) drain the other accumulator: bias,
// rotation, bf16, stored straight into the head layout.  The epilogue of tile
// j runs while the tensor core accumulates tile j + 1.
//
// rope_tables: cos / sin of p * base^(-2i/d) in fp64, rounded to fp32.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace infini {
namespace {

using namespace tc;

constexpr int kBM = 128;         // output rows (tokens) per tile
constexpr int kBN = 256;         // output columns per tile
constexpr int kBK = 64;          // d_model elements per ring stage (one swizzle panel)
constexpr int kStages = 4;
constexpr int kThreads = 192;    // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr uint32_t kABytes = kBM * kBK * 2;   // 16 KB
constexpr uint32_t kBBytes = kBN * kBK * 2;   // 32 KB
constexpr uint32_t kTmemCols = 2 * kBN;

struct ProjSmem {
  static constexpr uint32_t kA = 0;
  static constexpr uint32_t kB = kA + kStages * kABytes;
  static constexpr uint32_t kBar = kB + kStages * kBBytes;
  // full[kStages] empty[kStages] acc_full[2] acc_empty[2] drain
  static constexpr uint32_t kNumBars = 2 * kStages + 5;
  static constexpr uint32_t kBias = kBar + kNumBars * 8;        // the tile's bias [kBN] f32
  static constexpr uint32_t kTmemSlot = kBias + kBN * 4;
  static constexpr uint32_t kAbort = kTmemSlot + 4;
  static constexpr uint32_t kAlloc = kAbort + 4 + 1024;  // + room to align the base
  static_assert(kB % 1024 == 0 && kBar % 1024 == 0, "tiles must be 1024-byte aligned");
};

struct ProjArgs {
  __nv_bfloat16* q;
  __nv_bfloat16* k;
  __nv_bfloat16* v;
  const float* bias;   // [N] or null
  const float* rcos;   // [L][d/2] or null (no rotation)
  const float* rsin;
  unsigned int* status;
  int rows;            // B * L
  int n_out;           // (H_q + 2 H_kv) d
  int L, H_q, H_kv;
  int kslices;         // ceil(d_model / 64)
  int n_tiles, tiles;
};

__device__ __forceinline__ void load16f(const float* p, float* r) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(p) + i);
    r[4 * i] = v.x;
    r[4 * i + 1] = v.y;
    r[4 * i + 2] = v.z;
    r[4 * i + 3] = v.w;
  }
}

// Barrier `id` over `threads` threads (whole warps) that also returns whether
// any of them passed pred = true.
__device__ __forceinline__ bool named_barrier_or(int id, int threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void store16bf(__nv_bfloat16* dst, const float* x) {
  uint4 a, b;
  a.x = pack_bf16x2(x[0], x[1]);
  a.y = pack_bf16x2(x[2], x[3]);
  a.z = pack_bf16x2(x[4], x[5]);
  a.w = pack_bf16x2(x[6], x[7]);
  b.x = pack_bf16x2(x[8], x[9]);
  b.y = pack_bf16x2(x[10], x[11]);
  b.z = pack_bf16x2(x[12], x[13]);
  b.w = pack_bf16x2(x[14], x[15]);
  reinterpret_cast<uint4*>(dst)[0] = a;
  reinterpret_cast<uint4*>(dst)[1] = b;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
qkv_rope(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap tw,
         const ProjArgs a) {
  static_assert(kBN % D == 0 && D % 32 == 0, "a tile holds whole heads");
  constexpr int kHalf = D / 2;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ProjSmem::kBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* acc_full = bars + 2 * kStages;  // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + ProjSmem::kTmemSlot);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + ProjSmem::kAbort);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Copies and MMAs are issued under elect.sync; their commits must come from
  // the issuing thread, so the elected lane has to be the same every time.
  if (__syncthreads_or(elected_lane() != 0)) {
    if (threadIdx.x == 0) atomicOr(a.status, kStatusLayout);
    return;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full + i, 1);
      mbar_init(acc_empty + i, 4);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
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
    // ---------------------------------------------- TMA producer
    int it = 0;  // K slices issued so far (all tiles)
    bool ok = true;
    for (int t = blockIdx.x; ok && t < a.tiles; t += gridDim.x) {
      const int m0 = (t / a.n_tiles) * kBM, n0 = (t % a.n_tiles) * kBN;
      for (int kc = 0; kc < a.kslices; ++kc, ++it) {
        const int st = it % kStages;
        const uint32_t ph = (uint32_t)(it / kStages) & 1u;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(empty + st, ph ^ 1u, abort, a.status)))) break;
        if (elect_one()) {
          mbar_arrive_expect_tx(full + st, kABytes + kBBytes);
          tma_load_3d(smem + ProjSmem::kA + st * kABytes, &tx, full + st, kc * kBK, m0, 0);
          tma_load_3d(smem + ProjSmem::kB + st * kBBytes, &tw, full + st, kc * kBK, n0, 0);
        }
        __syncwarp();
      }
    }
    // Every copy issued must land before the CTA exits.
    for (int i = max(0, it - kStages); i < it; ++i)
      mbar_wait(full + i % kStages, (uint32_t)(i / kStages) & 1u, abort, a.status, false);
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------- MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, false, false);
    const uint64_t da = sw128_desc(smem_u32(smem + ProjSmem::kA), 16, 1024);
    const uint64_t db = sw128_desc(smem_u32(smem + ProjSmem::kB), 16, 1024);
    bool ok = true;
    int it = 0, j = 0;  // K slices and tiles so far
    for (int t = blockIdx.x; ok && t < a.tiles; t += gridDim.x, ++j) {
      const int acc = j & 1;
      // Accumulator acc is free once the epilogue has read tile j - 2.
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(acc_empty + acc, ((uint32_t)(j >> 1) & 1u) ^ 1u,
                                                    abort, a.status))))
        break;
      const uint32_t dacc = tmem + (uint32_t)(acc * kBN);
      for (int kc = 0; kc < a.kslices; ++kc, ++it) {
        const int st = it % kStages;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(full + st, (uint32_t)(it / kStages) & 1u, abort,
                                                      a.status))))
          break;
        tc_fence_after();
        if (elect_one()) {
          const uint64_t sa = da + ((st * kABytes) >> 4);
          const uint64_t sb = db + ((st * kBBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_ss(dacc, sa + kmajor_step(kk, kBM), sb + kmajor_step(kk, kBN), idesc,
                   (kc > 0 || kk > 0) ? 1u : 0u);
          tc_commit(empty + st);
          if (kc == a.kslices - 1) tc_commit(acc_full + acc);
        }
        __syncwarp();
      }
    }
    // Every MMA issued must complete before TMEM is released.
    if (elect_one()) tc_commit(drain);
    __syncwarp();
    mbar_wait(drain, 0, abort, a.status, false);
    __syncwarp();
  } else {
    // ---------------------------------------------- epilogue warps
    // Warp w reads TMEM lanes 32 (w % 4) .. + 31: row 32 (w % 4) + lane of
    // the tile.  Chunk-major: the rotation's cos / sin of a 16-column chunk
    // are loaded once per row and serve every query and key head of the
    // tile; the tile's bias sits in shared memory.  (Head-major order with
    // the bias and the tables read per head left two dependent global loads
    // in every step and made the epilogue, not the MMAs, the bound when the
    // contraction is short.)
    const int quarter = warp & 3;
    const uint32_t lq = (uint32_t)(32 * quarter) << 16;
    const int H_tot = a.H_q + 2 * a.H_kv;
    float* sbias = reinterpret_cast<float*>(smem + ProjSmem::kBias);
    const int et = threadIdx.x - 64;  // 0..127 over the four epilogue warps
    int j = 0;
    for (int t = blockIdx.x; t < a.tiles; t += gridDim.x, ++j) {
      const int acc = j & 1;
      const int m0 = (t / a.n_tiles) * kBM, n0 = (t % a.n_tiles) * kBN;
      const bool ok = __all_sync(0xffffffffu,
                                 mbar_wait(acc_full + acc, (uint32_t)(j >> 1) & 1u, abort, a.status));
      // The four epilogue warps leave together if any wait gave up (so that
      // none is left at a barrier); otherwise the previous tile's bias
      // readers are done, and this tile's bias is staged.
      if (named_barrier_or(1, 128, !ok)) break;
      for (int i = et; i < kBN; i += 128)
        sbias[i] = (a.bias != nullptr && n0 + i < a.n_out) ? __ldg(a.bias + n0 + i) : 0.f;
      named_barrier(1, 128);
      tc_fence_after();
      const int r = m0 + 32 * quarter + lane;
      const bool valid = r < a.rows;
      const int b = valid ? r / a.L : 0, tok = valid ? r - b * a.L : 0;
      const uint32_t tacc = tmem + (uint32_t)(acc * kBN) + lq;
      const int nh = min(kBN / D, H_tot - n0 / D);  // heads in this tile
      const bool tile_rot = a.rcos != nullptr && n0 / D < a.H_q + a.H_kv;
#pragma unroll
      for (int c = 0; c < kHalf; c += 16) {
        float cs[16], sn[16];
        if (tile_rot && valid) {
          load16f(a.rcos + (size_t)tok * kHalf + c, cs);
          load16f(a.rsin + (size_t)tok * kHalf + c, sn);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) cs[i] = 1.f, sn[i] = 0.f;
        }
#pragma unroll 1
        for (int hh = 0; hh < nh; ++hh) {
          const int gh = n0 / D + hh;  // head index over [q heads | k heads | v heads]
          __nv_bfloat16* base;
          int head, heads;
          if (gh < a.H_q) {
            base = a.q, head = gh, heads = a.H_q;
          } else if (gh < a.H_q + a.H_kv) {
            base = a.k, head = gh - a.H_q, heads = a.H_kv;
          } else {
            base = a.v, head = gh - a.H_q - a.H_kv, heads = a.H_kv;
          }
          const bool rot = a.rcos != nullptr && gh < a.H_q + a.H_kv;
          __nv_bfloat16* dst = base + (((size_t)b * heads + head) * a.L + tok) * D;
          uint32_t ulo[16], uhi[16];
          tmem_ld16(tacc + (uint32_t)(hh * D + c), ulo);
          tmem_ld16(tacc + (uint32_t)(hh * D + kHalf + c), uhi);
          tmem_wait_ld();
          float xl[16], xh[16];
          const float* bl = sbias + hh * D + c;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            xl[i] = __uint_as_float(ulo[i]) + bl[i];
            xh[i] = __uint_as_float(uhi[i]) + bl[kHalf + i];
          }
          if (rot) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float l = xl[i], u = xh[i];
              xl[i] = fmaf(l, cs[i], -u * sn[i]);
              xh[i] = fmaf(u, cs[i], l * sn[i]);
            }
          }
          if (valid) {
            store16bf(dst + c, xl);
            store16bf(dst + kHalf + c, xh);
          }
        }
      }
      // Accumulator acc may be overwritten once every warp has read it.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty + acc);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// cos / sin of p * base^(-2i/d), p = 0..n_pos-1, i < d/2, computed in fp64.
__global__ void rope_tables_kernel(float* __restrict__ cos_out, float* __restrict__ sin_out,
                                   int n_pos, int half, int d, double base) {
  const size_t n = (size_t)n_pos * half;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (size_t)gridDim.x * blockDim.x) {
    const int p = (int)(e / half), i = (int)(e % half);
    const double ang = (double)p * pow(base, -2.0 * i / d);
    double s, c;
    sincos(ang, &s, &c);
    cos_out[e] = (float)c;
    sin_out[e] = (float)s;
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

// 2-D bf16 matrix [rows][cols] (cols contiguous) as a 3-D map with one plane;
// box 64 x box_rows, 128-byte swizzle; out-of-range elements read as zero.
bool make_matrix_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows,
                     uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {cols, rows, 1};
  cuuint64_t strides[2] = {cols * 2, cols * rows * 2};
  cuuint32_t box[3] = {(cuuint32_t)kBK, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch(const ProjectionProblem& p, cudaStream_t stream) {
  const long long rows = (long long)p.B * p.L;
  const long long N = (long long)(p.H_q + 2 * p.H_kv) * D;
  CUtensorMap tx, tw;
  if (!make_matrix_map(&tx, p.x, (uint64_t)p.d_model, (uint64_t)rows, kBM) ||
      !make_matrix_map(&tw, p.w, (uint64_t)p.d_model, (uint64_t)N, kBN))
    return cudaErrorInvalidValue;
  ProjArgs a;
  a.q = static_cast<__nv_bfloat16*>(p.q);
  a.k = static_cast<__nv_bfloat16*>(p.k);
  a.v = static_cast<__nv_bfloat16*>(p.v);
  a.bias = p.bias;
  a.rcos = p.rope_cos;
  a.rsin = p.rope_sin;
  a.status = p.status;
  a.rows = (int)rows;
  a.n_out = (int)N;
  a.L = p.L;
  a.H_q = p.H_q;
  a.H_kv = p.H_kv;
  a.kslices = (p.d_model + kBK - 1) / kBK;
  a.n_tiles = (int)((N + kBN - 1) / kBN);
  const long long tiles = ((rows + kBM - 1) / kBM) * (long long)a.n_tiles;
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  a.tiles = (int)tiles;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int grid = a.tiles < sms ? a.tiles : sms;  // persistent: one CTA per SM
  auto kern = qkv_rope<D>;
  if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)ProjSmem::kAlloc)) != cudaSuccess)
    return e;
  kern<<<grid, kThreads, ProjSmem::kAlloc, stream>>>(tx, tw, a);
  return cudaGetLastError();
}

}  // namespace

bool qkv_projection_supported(int d_k, int d_v, int d_model, bool bf16) {
  return bf16 && d_k == d_v && (d_k == 64 || d_k == 128) && d_model >= kBK && d_model % 8 == 0;
}

cudaError_t launch_qkv_projection(const ProjectionProblem& p, cudaStream_t stream) {
  if (p.d == 128) return launch<128>(p, stream);
  if (p.d == 64) return launch<64>(p, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_rope_tables(float* cos_out, float* sin_out, int n_pos, int d, double base,
                               cudaStream_t stream) {
  const size_t n = (size_t)n_pos * (d / 2);
  const size_t blocks = (n + 255) / 256;
  const unsigned grid = (unsigned)(blocks < 4096 ? blocks : 4096);
  rope_tables_kernel<<<grid, 256, 0, stream>>>(cos_out, sin_out, n_pos, d / 2, d, base);
  return cudaGetLastError();
}

}  // namespace infini
