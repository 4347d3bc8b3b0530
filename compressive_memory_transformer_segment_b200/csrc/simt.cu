// fp32 CUDA-core kernels for the Infini-attention forward.
//
// These are the exact-arithmetic path: every product and sum is fp32, so the
// fp32-I/O configuration meets a 1e-4 tolerance.  They run any segment length
// and any supported head size, and serve bf16 I/O where the tensor-core path
// does not apply.
//
//   simt_state_scan : per KV head, scans the segments in order and writes the
//                     memory each segment reads, (M_{s-1}, z_{s-1}), to the
//                     workspace, then (M_T, z_T) to the outputs
//                     ("Hugging Face Infini-Attention 再現分析", Memory Update
//                     and State Transfer; "Leave No Context Behind"
//                     explainer, "メモリの更新" incl. the delta rule).
//   simt_attention  : per (query tile, segment, head, batch): local causal
//                     softmax attention, retrieval from (M_{s-1}, z_{s-1}) and
//                     the beta gate (Local Attention, Memory Retrieval,
//                     Integration; "実装上の流れ").
#include "common.cuh"
#include "kernels.h"

namespace infini {

namespace {

constexpr int kScanThreads = 256;
constexpr int kScanChunk = 32;   // tokens staged in shared memory per step
constexpr int kScanCols = 32;    // columns of M owned by one CTA

// Shared-memory plan of the scan (floats).
template <int DK>
struct ScanSmem {
  static constexpr int kSkStride = DK + 4;  // rows of sigma(K); +4 spreads banks
  static constexpr int kSk = kScanChunk * kSkStride;
  static constexpr int kMs = DK * kScanCols;     // M_{s-1}[:, cols] (delta)
  static constexpr int kUs = kScanChunk * kScanCols;
  static constexpr int kZ = DK;                  // z_{s-1}
  static constexpr int kDz = DK;                 // this segment's sum of sigma(K)
  static constexpr int kRden = kScanChunk;
  static constexpr int kTotal = kSk + kMs + kUs + kZ + kDz + kRden;
};

// Grid: (d_v / 32, B * H_kv).  CTA (cb, bh) owns columns [32 cb, 32 cb + 32)
// of the chain's M for the whole scan; the delta rule's column j depends only
// on column j of M and on the shared denominator sigma(K) z, so the column
// blocks are independent.  Thread (warp w, lane c) holds M[w + 8 i][c].
template <typename T, typename MP, int DK, int DV, bool DELTA>
__global__ void __launch_bounds__(kScanThreads)
simt_state_scan(const T* __restrict__ kx, const T* __restrict__ vx,
                const float* __restrict__ M_in, float* __restrict__ M_out,
                float* __restrict__ z_out, float* __restrict__ z_pref,
                MP* __restrict__ M_pref, int L, int S, int nseg, int BH) {
  using SM = ScanSmem<DK>;
  extern __shared__ float smem[];
  float* sK = smem;
  float* Ms = sK + SM::kSk;
  float* Us = Ms + SM::kMs;
  float* zs = Us + SM::kUs;
  float* dz = zs + SM::kZ;
  float* rden = dz + SM::kDz;

  constexpr int kRows = DK / 8;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c0 = blockIdx.x * kScanCols;
  const int bh = blockIdx.y;
  const T* kc = kx + (size_t)bh * L * DK;
  const T* vc = vx + (size_t)bh * L * DV;

  float Mreg[kRows], dM[kRows];
#pragma unroll
  for (int i = 0; i < kRows; ++i)
    Mreg[i] = M_in[((size_t)bh * DK + warp + 8 * i) * DV + c0 + lane];
  // z_in was copied to slot 0 of z_pref before this kernel.
  for (int kk = tid; kk < DK; kk += kScanThreads) zs[kk] = z_pref[(size_t)bh * DK + kk];
  __syncthreads();

  for (int s = 0; s < nseg; ++s) {
    const int r0 = s * S;
    const int r1 = min(r0 + S, L);
    // The memory segment s reads: M_{s-1}, z_{s-1}.
    MP* Mp = M_pref + ((size_t)s * BH + bh) * DK * DV;
#pragma unroll
    for (int i = 0; i < kRows; ++i) {
      Mp[(size_t)(warp + 8 * i) * DV + c0 + lane] = from_f32<MP>(Mreg[i]);
      dM[i] = 0.f;
      if (DELTA) Ms[(warp + 8 * i) * kScanCols + lane] = Mreg[i];
    }
    if (blockIdx.x == 0 && s > 0)
      for (int kk = tid; kk < DK; kk += kScanThreads)
        z_pref[((size_t)s * BH + bh) * DK + kk] = zs[kk];
    for (int kk = tid; kk < DK; kk += kScanThreads) dz[kk] = 0.f;

    for (int t0 = r0; t0 < r1; t0 += kScanChunk) {
      __syncthreads();  // previous chunk fully consumed
      // Stage sigma(K) (rows past the segment end are 0) and V[:, cols].
      for (int e = tid; e < kScanChunk * DK; e += kScanThreads) {
        const int t = e / DK, kk = e % DK;
        const int row = t0 + t;
        sK[t * SM::kSkStride + kk] = row < r1 ? elu1(to_f32(kc[(size_t)row * DK + kk])) : 0.f;
      }
      for (int e = tid; e < kScanChunk * kScanCols; e += kScanThreads) {
        const int t = e / kScanCols, c = e % kScanCols;
        const int row = t0 + t;
        Us[e] = row < r1 ? to_f32(vc[(size_t)row * DV + c0 + c]) : 0.f;
      }
      __syncthreads();
      if (DELTA) {
        // U = V - sigma(K) M_{s-1} / (sigma(K) z_{s-1}); thread -> (t, 4 columns).
        const int t = tid >> 3, cq = (tid & 7) * 4;
        float r[4] = {0.f, 0.f, 0.f, 0.f};
        float den = 0.f;
        const float* sk = sK + t * SM::kSkStride;
#pragma unroll 8
        for (int kk = 0; kk < DK; ++kk) {
          const float a = sk[kk];
          const float4 m = *reinterpret_cast<const float4*>(Ms + kk * kScanCols + cq);
          r[0] = fmaf(a, m.x, r[0]);
          r[1] = fmaf(a, m.y, r[1]);
          r[2] = fmaf(a, m.z, r[2]);
          r[3] = fmaf(a, m.w, r[3]);
          den = fmaf(a, zs[kk], den);
        }
        __syncthreads();  // everyone has read V from Us
        if (t0 + t < r1) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float ret = den != 0.f ? r[j] / den : 0.f;
            Us[t * kScanCols + cq + j] -= ret;
          }
        }
        __syncthreads();
      }
      // dM[k][c] += sum_t sigma(K)[t][k] * U[t][c];  dz[k] += sum_t sigma(K)[t][k].
      const int tmax = min(kScanChunk, r1 - t0);
      for (int t = 0; t < tmax; ++t) {
        const float u = Us[t * kScanCols + lane];
        const float* sk = sK + t * SM::kSkStride;
#pragma unroll
        for (int i = 0; i < kRows; ++i) dM[i] = fmaf(sk[warp + 8 * i], u, dM[i]);
      }
      for (int kk = tid; kk < DK; kk += kScanThreads) {
        float acc = 0.f;
        for (int t = 0; t < tmax; ++t) acc += sK[t * SM::kSkStride + kk];
        dz[kk] += acc;
      }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kRows; ++i) Mreg[i] += dM[i];
    for (int kk = tid; kk < DK; kk += kScanThreads) zs[kk] += dz[kk];
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < kRows; ++i)
    M_out[((size_t)bh * DK + warp + 8 * i) * DV + c0 + lane] = Mreg[i];
  if (blockIdx.x == 0)
    for (int kk = tid; kk < DK; kk += kScanThreads) z_out[(size_t)bh * DK + kk] = zs[kk];
}

constexpr int kAttThreads = 256;
constexpr int kBQ = 64;  // query rows per CTA (8 warps x 8 rows)
constexpr int kBK = 64;  // keys per shared-memory tile

template <int DK, int DV>
struct AttSmem {
  static constexpr int kKStride = DK + 1;
  static constexpr int kQ = kBQ * DK;
  static constexpr int kK = kBK * kKStride;
  static constexpr int kV = kBK * DV;
  static constexpr int kMem = DK * DV + DK;  // M_{s-1} and z_{s-1}, reusing K/V space
  static constexpr int kKV = (kK + kV) > kMem ? (kK + kV) : kMem;
  static constexpr int kTotal = kQ + kKV;
};

// Grid: (query tiles over the whole sequence, B * H_q).  Query tiles never
// straddle a segment: a segment of n rows has ceil(n / 64) tiles.
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kAttThreads)
simt_attention(const T* __restrict__ qx, const T* __restrict__ kx, const T* __restrict__ vx,
               const float* __restrict__ beta, const float* __restrict__ M_pref,
               const float* __restrict__ z_pref, T* __restrict__ out, int H_q, int H_kv,
               int L, int S, int tiles_per_seg) {
  using SM = AttSmem<DK, DV>;
  extern __shared__ float smem[];
  float* Qs = smem;
  float* Ks = Qs + SM::kQ;
  float* Vs = Ks + SM::kK;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bhq = blockIdx.y;
  const int b = bhq / H_q, h = bhq % H_q;
  const int g = H_q / H_kv;
  const int bh = b * H_kv + h / g;
  const int BH = gridDim.y / g;  // = B * H_kv
  const int s = blockIdx.x / tiles_per_seg;
  const int qt = blockIdx.x % tiles_per_seg;
  const int seg0 = s * S;
  const int seg_len = min(S, L - seg0);
  const int q0 = qt * kBQ;  // first local row of this tile
  if (q0 >= seg_len) return;  // tile past a short last segment
  const int q_hi = min(q0 + kBQ, seg_len) - 1;

  const T* qc = qx + ((size_t)bhq * L + seg0) * DK;
  const T* kc = kx + ((size_t)bh * L + seg0) * DK;
  const T* vc = vx + ((size_t)bh * L + seg0) * DV;

  for (int e = tid; e < kBQ * DK; e += kAttThreads) {
    const int r = e / DK;
    Qs[e] = (q0 + r < seg_len) ? to_f32(qc[(size_t)(q0 + r) * DK + (e % DK)]) : 0.f;
  }

  constexpr int kRowsPerWarp = kBQ / 8;
  constexpr int kCols = DV / 32;
  const float scale = rsqrtf((float)DK) * 1.4426950408889634f;  // softmax in base 2
  float m[kRowsPerWarp], l[kRowsPerWarp], o[kRowsPerWarp][kCols];
#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr) {
    m[rr] = -INFINITY;
    l[rr] = 0.f;
#pragma unroll
    for (int c = 0; c < kCols; ++c) o[rr][c] = 0.f;
  }

  for (int k0 = 0; k0 <= q_hi; k0 += kBK) {
    __syncthreads();
    for (int e = tid; e < kBK * DK; e += kAttThreads) {
      const int j = e / DK, kk = e % DK;
      Ks[j * SM::kKStride + kk] = (k0 + j < seg_len) ? to_f32(kc[(size_t)(k0 + j) * DK + kk]) : 0.f;
    }
    for (int e = tid; e < kBK * DV; e += kAttThreads) {
      const int j = e / DV;
      Vs[e] = (k0 + j < seg_len) ? to_f32(vc[(size_t)(k0 + j) * DV + (e % DV)]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
      const int i = q0 + warp * kRowsPerWarp + rr;  // local query row
      const float* qi = Qs + (warp * kRowsPerWarp + rr) * DK;
      const float* ka = Ks + lane * SM::kKStride;
      const float* kb = Ks + (lane + 32) * SM::kKStride;
      float sa = 0.f, sb = 0.f;
#pragma unroll 8
      for (int kk = 0; kk < DK; ++kk) {
        const float qv = qi[kk];
        sa = fmaf(qv, ka[kk], sa);
        sb = fmaf(qv, kb[kk], sb);
      }
      sa = (k0 + lane <= i) ? sa * scale : -INFINITY;
      sb = (k0 + lane + 32 <= i) ? sb * scale : -INFINITY;
      const float m_new = fmaxf(m[rr], warp_max(fmaxf(sa, sb)));
      if (m_new == -INFINITY) continue;  // row sees no key in this tile yet
      const float alpha = exp2f(m[rr] - m_new);
      const float pa = exp2f(sa - m_new), pb = exp2f(sb - m_new);
      l[rr] = l[rr] * alpha + warp_sum(pa + pb);
      m[rr] = m_new;
#pragma unroll
      for (int c = 0; c < kCols; ++c) o[rr][c] *= alpha;
#pragma unroll 4
      for (int j = 0; j < 32; ++j) {
        const float wa = __shfl_sync(0xffffffffu, pa, j);
        const float wb = __shfl_sync(0xffffffffu, pb, j);
#pragma unroll
        for (int c = 0; c < kCols; ++c) {
          o[rr][c] = fmaf(wa, Vs[j * DV + lane + 32 * c], o[rr][c]);
          o[rr][c] = fmaf(wb, Vs[(j + 32) * DV + lane + 32 * c], o[rr][c]);
        }
      }
    }
  }

  // Retrieval from the memory this segment reads: M_{s-1}, z_{s-1}.
  __syncthreads();
  float* Ms = Ks;
  float* zs = Ms + DK * DV;
  const float* Mg = M_pref + ((size_t)s * BH + bh) * DK * DV;
  for (int e = tid; e < DK * DV; e += kAttThreads) Ms[e] = Mg[e];
  for (int e = tid; e < DK; e += kAttThreads) zs[e] = z_pref[((size_t)s * BH + bh) * DK + e];
  for (int e = tid; e < kBQ * DK; e += kAttThreads) Qs[e] = elu1(Qs[e]);
  __syncthreads();

  const float gm = gate_sigmoid(beta[h]);
  T* oc = out + ((size_t)bhq * L + seg0) * DV;
#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr) {
    const int i = q0 + warp * kRowsPerWarp + rr;
    if (i >= seg_len) continue;
    const float* sq = Qs + (warp * kRowsPerWarp + rr) * DK;
    float num[kCols];
#pragma unroll
    for (int c = 0; c < kCols; ++c) num[c] = 0.f;
    float den = 0.f;
#pragma unroll 4
    for (int kk = 0; kk < DK; ++kk) {
      const float a = sq[kk];
      den = fmaf(a, zs[kk], den);
#pragma unroll
      for (int c = 0; c < kCols; ++c) num[c] = fmaf(a, Ms[kk * DV + lane + 32 * c], num[c]);
    }
    const float inv_l = 1.f / l[rr];
#pragma unroll
    for (int c = 0; c < kCols; ++c) {
      const float a_mem = den != 0.f ? num[c] / den : 0.f;
      const float a_dot = o[rr][c] * inv_l;
      oc[(size_t)i * DV + lane + 32 * c] = from_f32<T>(gm * a_mem + (1.f - gm) * a_dot);
    }
  }
}

template <typename T, int DK, int DV>
cudaError_t scan_dispatch_rule(const Problem& p, cudaStream_t stream) {
  const size_t smem = ScanSmem<DK>::kTotal * sizeof(float);
  dim3 grid(DV / kScanCols, p.B * p.H_kv);
  if (p.M_pref_bf16) {
    auto kern = p.delta ? simt_state_scan<T, __nv_bfloat16, DK, DV, true>
                        : simt_state_scan<T, __nv_bfloat16, DK, DV, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kScanThreads, smem, stream>>>(
        static_cast<const T*>(p.k), static_cast<const T*>(p.v), p.M_in, p.M_out, p.z_out,
        p.z_pref, static_cast<__nv_bfloat16*>(p.M_pref), p.L, p.S, p.T, p.B * p.H_kv);
    return cudaGetLastError();
  }
  auto kern = p.delta ? simt_state_scan<T, float, DK, DV, true> : simt_state_scan<T, float, DK, DV, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kScanThreads, smem, stream>>>(
      static_cast<const T*>(p.k), static_cast<const T*>(p.v), p.M_in, p.M_out, p.z_out,
      p.z_pref, static_cast<float*>(p.M_pref), p.L, p.S, p.T, p.B * p.H_kv);
  return cudaGetLastError();
}

template <typename T, int DK, int DV>
cudaError_t att_dispatch(const Problem& p, cudaStream_t stream) {
  const size_t smem = AttSmem<DK, DV>::kTotal * sizeof(float);
  const int tps = (p.S + kBQ - 1) / kBQ;
  dim3 grid((unsigned)(tps * p.T), p.B * p.H_q);
  auto kern = simt_attention<T, DK, DV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kAttThreads, smem, stream>>>(
      static_cast<const T*>(p.q), static_cast<const T*>(p.k), static_cast<const T*>(p.v), p.beta,
      static_cast<const float*>(p.M_pref), p.z_pref, static_cast<T*>(p.out), p.H_q, p.H_kv, p.L,
      p.S, tps);
  return cudaGetLastError();
}

#define INFINI_DIM_SWITCH(FN, T, p, stream)                                   \
  switch (p.d_k * 1000 + p.d_v) {                                             \
    case 32032: return FN<T, 32, 32>(p, stream);                              \
    case 32064: return FN<T, 32, 64>(p, stream);                              \
    case 32128: return FN<T, 32, 128>(p, stream);                             \
    case 64032: return FN<T, 64, 32>(p, stream);                              \
    case 64064: return FN<T, 64, 64>(p, stream);                              \
    case 64128: return FN<T, 64, 128>(p, stream);                             \
    case 128032: return FN<T, 128, 32>(p, stream);                            \
    case 128064: return FN<T, 128, 64>(p, stream);                            \
    case 128128: return FN<T, 128, 128>(p, stream);                           \
    default: return cudaErrorInvalidValue;                                    \
  }

}  // namespace

cudaError_t launch_simt_state_scan(const Problem& p, cudaStream_t stream) {
  if (p.bf16) { INFINI_DIM_SWITCH(scan_dispatch_rule, __nv_bfloat16, p, stream) }
  INFINI_DIM_SWITCH(scan_dispatch_rule, float, p, stream)
}

cudaError_t launch_simt_attention(const Problem& p, cudaStream_t stream) {
  if (p.bf16) { INFINI_DIM_SWITCH(att_dispatch, __nv_bfloat16, p, stream) }
  INFINI_DIM_SWITCH(att_dispatch, float, p, stream)
}

}  // namespace infini
