// Streaming decode step of the Infini-attention layer (sm_100a, CUDA cores).
//
// One call takes one new token per (batch row, head): its query q_t, key k_t
// and value v_t.  The current segment's keys and values so far sit in a
// rolling buffer of S rows per KV head; the new token goes to row `pos`, and
// its output is the same as the layer forward gives that token:
//   A_dot = softmax over buffer rows 0..pos of q_t . k_j / sqrt(d), times V
//           (causal: the token sees itself and the earlier tokens of its
//           segment; "Hugging Face Infini-Attention 再現分析", Local Attention),
//   A_mem = sigma(q_t) M_{s-1} / (sigma(q_t) z_{s-1}), 0 where the denominator
//           is 0 (Memory Retrieval),
//   out_t = sg(beta_h) A_mem + (1 - sg(beta_h)) A_dot (Integration).
// When the token fills the segment (pos = S - 1), the memory is updated with
// the whole buffer by the forward's own scan kernels (Memory Update, State
// Transfer): the caller of this launcher does that after it.
//
// Decode is bound by memory traffic and latency (each buffer row and M are
// read once per step, a few flops per byte), so it runs on CUDA cores, in
// ONE kernel per step: grid (row chunks + 1, B * H_kv, query-head chunks).
//   - CTA x < chunks: up to kRows (64) buffer rows of one KV head, read once
//     for up to kG query heads of its group.  A warp takes 8 rows at a time (vector
//     loads, lanes across d; the 8 x kG dot products and their 2^x are
//     independent, so the latency of one row overlaps the next), keeping an
//     online softmax per head; the CTA's partial (max, sum, acc[d]) per head
//     goes to the workspace.  The CTA whose chunk holds row `pos` takes that
//     row from k_t, v_t and stores it in the buffer.
//   - CTA x = chunks: the retrieval of those heads, sigma(q) M and sigma(q).z,
//     reading M once for the group (warps split M's rows, lanes its columns).
//   - Each CTA then takes a ticket from the group's counter; the last one
//     merges the partials with the retrieval and the gate and stores out_t,
//     then puts the counter back to 0.  No CTA waits for another.
#include "common.cuh"
#include "kernels.h"

namespace infini {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kG = 4;           // query heads per CTA
constexpr int kNB = 8;          // rows per warp (one batch: all its loads in flight at once)
constexpr int kRows = kWarps * kNB;  // buffer rows per attention CTA

// Raw vector of E elements of T (E * sizeof(T) = 2, 4, 8 or 16 bytes).
template <int BYTES> struct RawVec;
template <> struct RawVec<2> { using type = unsigned short; };
template <> struct RawVec<4> { using type = unsigned int; };
template <> struct RawVec<8> { using type = uint2; };
template <> struct RawVec<16> { using type = uint4; };

template <typename T, int E>
using Raw = typename RawVec<E * (int)sizeof(T)>::type;

template <typename T, int E>
__device__ __forceinline__ Raw<T, E> load_raw(const T* p) {
  return *reinterpret_cast<const Raw<T, E>*>(p);
}

// Element i of a raw vector as a float.
template <typename T, int E>
__device__ __forceinline__ float elem(const Raw<T, E>& raw, int i) {
  return to_f32<T>(reinterpret_cast<const T*>(&raw)[i]);
}

template <typename T, int E>
__device__ __forceinline__ void copy_vec(const T* src, T* dst) {
  using V = typename RawVec<E * (int)sizeof(T)>::type;
  *reinterpret_cast<V*>(dst) = *reinterpret_cast<const V*>(src);
}

// Sums each of v[0..31] over the 32 lanes of the warp; afterwards every lane
// holds all 32 totals.  Recursive halving (each exchange sends half of the
// values still held, so that lane L ends with the total of value L: 31
// shuffles) and a broadcast back (32 shuffles), against 32 x 5 shuffles for
// 32 separate butterfly sums: the shuffle unit, not the arithmetic, bounds
// the step's 32 dot products per warp.
__device__ __forceinline__ void warp_sum32(float (&v)[32], int lane) {
  float w[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) w[i] = v[i];
#pragma unroll
  for (int lvl = 0; lvl < 5; ++lvl) {
    const int o = 16 >> lvl;  // lanes exchanged with, and values kept
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (i < o) {
        const float send = upper ? w[i] : w[i + o];
        const float keep = upper ? w[i + o] : w[i];
        w[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __shfl_sync(0xffffffffu, w[0], i);
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 2)
decode_step_kernel(DecodeProblem p) {
  static_assert(kNB * kG == 32, "one score per lane after the reduce-scatter");
  constexpr int E = D / 32;  // elements of d per lane
  __shared__ float qs[kG][D];
  __shared__ float red[kWarps][kG][D + 2];
  __shared__ int last;

  const int nch = (p.pos + kRows) / kRows;  // attention CTAs of the group
  const int c = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / p.H_kv, hk = bh - b * p.H_kv;
  const int g = p.H_q / p.H_kv;
  const int hq0 = hk * g + blockIdx.z * kG;
  const int ng = min(kG, g - (int)blockIdx.z * kG);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const T* q_t = static_cast<const T*>(p.q_t);

  if (c < nch) {
    // ------------------------------------------------ attention partial
    const int r0 = c * kRows, r1 = min(r0 + kRows, p.pos + 1);
    const T* k_t = static_cast<const T*>(p.k_t) + (size_t)bh * D;
    const T* v_t = static_cast<const T*>(p.v_t) + (size_t)bh * D;
    T* kbuf = static_cast<T*>(p.k_buf) + (size_t)bh * p.S * D;
    T* vbuf = static_cast<T*>(p.v_buf) + (size_t)bh * p.S * D;
    // Queries in base-2 units: q * log2(e) / sqrt(d).
    const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;
    for (int i = threadIdx.x; i < kG * D; i += kThreads) {
      const int hh = i / D, e = i - hh * D;
      qs[hh][e] = hh < ng ? to_f32<T>(q_t[(size_t)(b * p.H_q + hq0 + hh) * D + e]) * sl2 : 0.f;
    }
    __syncthreads();
    float qr[kG][E];
#pragma unroll
    for (int hh = 0; hh < kG; ++hh)
#pragma unroll
      for (int e = 0; e < E; ++e) qr[hh][e] = qs[hh][lane * E + e];

    float m[kG], l[kG], acc[kG][E];
#pragma unroll
    for (int hh = 0; hh < kG; ++hh) {
      m[hh] = -INFINITY;
      l[hh] = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[hh][e] = 0.f;
    }
    // This warp's rows: r0 + warp * kNB + i, i < nr (one batch).
    const int nr = max(0, min(kNB, r1 - r0 - warp * kNB));
    for (int i0 = 0; i0 < nr; i0 += kNB) {
      Raw<T, E> kx[kNB], vx[kNB];
#pragma unroll
      for (int rr = 0; rr < kNB; ++rr) {
        const int j = r0 + warp * kNB + i0 + rr;
        if (i0 + rr < nr) {
          const bool fresh = j == p.pos;
          const T* kr = (fresh ? k_t : kbuf + (size_t)j * D) + lane * E;
          const T* vr = (fresh ? v_t : vbuf + (size_t)j * D) + lane * E;
          kx[rr] = load_raw<T, E>(kr);
          vx[rr] = load_raw<T, E>(vr);
          if (fresh && blockIdx.z == 0) {
            copy_vec<T, E>(kr, kbuf + (size_t)j * D + lane * E);
            copy_vec<T, E>(vr, vbuf + (size_t)j * D + lane * E);
          }
        } else {
          kx[rr] = Raw<T, E>{};
          vx[rr] = Raw<T, E>{};
        }
      }
      float s[kNB][kG];
#pragma unroll
      for (int rr = 0; rr < kNB; ++rr)
#pragma unroll
        for (int hh = 0; hh < kG; ++hh) {
          float t = 0.f;
#pragma unroll
          for (int e = 0; e < E; ++e) t = fmaf(qr[hh][e], elem<T, E>(kx[rr], e), t);
          s[rr][hh] = t;
        }
      {
        float sv[32];
#pragma unroll
        for (int rr = 0; rr < kNB; ++rr)
#pragma unroll
          for (int hh = 0; hh < kG; ++hh) sv[rr * kG + hh] = s[rr][hh];
        warp_sum32(sv, lane);
#pragma unroll
        for (int rr = 0; rr < kNB; ++rr)
#pragma unroll
          for (int hh = 0; hh < kG; ++hh) s[rr][hh] = i0 + rr < nr ? sv[rr * kG + hh] : -INFINITY;
      }
#pragma unroll
      for (int hh = 0; hh < kG; ++hh) {
        float bm = s[0][hh];
#pragma unroll
        for (int rr = 1; rr < kNB; ++rr) bm = fmaxf(bm, s[rr][hh]);
        const float mn = fmaxf(m[hh], bm);      // finite: row i0 is valid
        const float corr = exp2f(m[hh] - mn);   // 0 on the first batch
        l[hh] *= corr;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[hh][e] *= corr;
#pragma unroll
        for (int rr = 0; rr < kNB; ++rr) {
          const float pj = exp2f(s[rr][hh] - mn);  // 0 for rows past the end
          l[hh] += pj;
#pragma unroll
          for (int e = 0; e < E; ++e) acc[hh][e] = fmaf(pj, elem<T, E>(vx[rr], e), acc[hh][e]);
        }
        m[hh] = mn;
      }
    }
    // Merge the warps' partials; one (max, sum, acc[d]) per head to the
    // workspace.
#pragma unroll
    for (int hh = 0; hh < kG; ++hh) {
      if (lane == 0) {
        red[warp][hh][D] = m[hh];
        red[warp][hh][D + 1] = l[hh];
      }
#pragma unroll
      for (int e = 0; e < E; ++e) red[warp][hh][lane * E + e] = acc[hh][e];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < ng * D; i += kThreads) {
      const int hh = i / D, e = i - hh * D;
      float mx = -INFINITY;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) mx = fmaxf(mx, red[w][hh][D]);
      float ls = 0.f, as = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        // A warp without rows has m = -inf, l = acc = 0; mx is finite.
        const float f = red[w][hh][D] == -INFINITY ? 0.f : exp2f(red[w][hh][D] - mx);
        ls = fmaf(red[w][hh][D + 1], f, ls);
        as = fmaf(red[w][hh][e], f, as);
      }
      float* part = p.part + ((size_t)(b * p.H_q + hq0 + hh) * p.nsplit + c) * (D + 2);
      part[2 + e] = as;
      if (e == 0) {
        part[0] = mx;
        part[1] = ls;
      }
    }
  } else {
    // ------------------------------------------------ retrieval
    // sigma(q) for the CTA's heads; den = sigma(q).z; num = sigma(q) M with
    // warp w summing M's rows [w D/4, (w+1) D/4) and lane l columns l + 32 cc.
    for (int i = threadIdx.x; i < kG * D; i += kThreads) {
      const int hh = i / D, e = i - hh * D;
      qs[hh][e] = hh < ng ? elu1(to_f32<T>(q_t[(size_t)(b * p.H_q + hq0 + hh) * D + e])) : 0.f;
    }
    __syncthreads();
    const float* zv = p.z + (size_t)bh * D;
    const float* Mh = p.M + (size_t)bh * D * D;
    if (warp < ng) {
      float dp = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) dp = fmaf(qs[warp][lane + 32 * e], zv[lane + 32 * e], dp);
      dp = warp_sum(dp);
      if (lane == 0) p.ret[(size_t)(b * p.H_q + hq0 + warp) * (D + 1) + D] = dp;
    }
    float nacc[kG][E];
#pragma unroll
    for (int hh = 0; hh < kG; ++hh)
#pragma unroll
      for (int cc = 0; cc < E; ++cc) nacc[hh][cc] = 0.f;
    constexpr int kRowsPerWarp = D / kWarps;
    const int i_0 = warp * kRowsPerWarp;
#pragma unroll 8
    for (int i = 0; i < kRowsPerWarp; ++i) {
      float mrow[E];
#pragma unroll
      for (int cc = 0; cc < E; ++cc) mrow[cc] = Mh[(size_t)(i_0 + i) * D + lane + 32 * cc];
#pragma unroll
      for (int hh = 0; hh < kG; ++hh) {
        const float sqv = qs[hh][i_0 + i];
#pragma unroll
        for (int cc = 0; cc < E; ++cc) nacc[hh][cc] = fmaf(sqv, mrow[cc], nacc[hh][cc]);
      }
    }
#pragma unroll
    for (int hh = 0; hh < kG; ++hh)
#pragma unroll
      for (int cc = 0; cc < E; ++cc) red[warp][hh][lane + 32 * cc] = nacc[hh][cc];
    __syncthreads();
    for (int i = threadIdx.x; i < ng * D; i += kThreads) {
      const int hh = i / D, e = i - hh * D;
      float num = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) num += red[w][hh][e];
      p.ret[(size_t)(b * p.H_q + hq0 + hh) * (D + 1) + e] = num;
    }
  }

  // ------------------------------------------------ the last CTA finishes
  __threadfence();  // this thread's workspace writes, before the ticket
  __syncthreads();
  unsigned int* ctr = p.ctr + (size_t)bh * gridDim.z + blockIdx.z;
  if (threadIdx.x == 0) last = atomicAdd(ctr, 1u) == (unsigned int)nch;
  __syncthreads();
  if (!last) return;
  __threadfence();  // every other CTA's writes of this group are visible
  // The retrieval terms and the gates of this thread's output column, loaded
  // now so that they arrive during the merge of the partials.
  float r_num[kG], r_den[kG], gate[kG];
  {
    const int e = threadIdx.x % D;
#pragma unroll
    for (int hh = 0; hh < kG; ++hh) {
      const bool ok = hh < ng && threadIdx.x < D;
      const float* rt = p.ret + (size_t)(b * p.H_q + hq0 + (ok ? hh : 0)) * (D + 1);
      r_num[hh] = ok ? __ldcg(rt + e) : 0.f;
      r_den[hh] = ok ? __ldcg(rt + D) : 0.f;
      gate[hh] = ok ? p.beta[hq0 + hh] : 0.f;
    }
  }
  // Column e of every head of the CTA is merged by kParts threads, each over
  // every kParts-th chunk, four chunks at a time for all heads (independent
  // loads in flight) with a running max; then the parts are combined.
  constexpr int kParts = kThreads / D;
  {
    const int e = threadIdx.x % D, part_id = threadIdx.x / D;
    constexpr int kU = 4;
    float mx[kG], ls[kG], as[kG];
#pragma unroll
    for (int hh = 0; hh < kG; ++hh) {
      mx[hh] = -INFINITY;
      ls[hh] = 0.f;
      as[hh] = 0.f;
    }
    for (int c0 = part_id; c0 < nch; c0 += kU * kParts) {
      float mc[kG][kU], lc[kG][kU], ac[kG][kU];
#pragma unroll
      for (int hh = 0; hh < kG; ++hh) {
        const float* part = p.part + (size_t)(b * p.H_q + hq0 + hh) * p.nsplit * (D + 2);
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int cc = c0 + u * kParts;
          const bool ok = hh < ng && cc < nch;
          const float* pc = part + (size_t)cc * (D + 2);
          mc[hh][u] = ok ? __ldcg(pc) : -INFINITY;
          lc[hh][u] = ok ? __ldcg(pc + 1) : 0.f;
          ac[hh][u] = ok ? __ldcg(pc + 2 + e) : 0.f;
        }
      }
#pragma unroll
      for (int hh = 0; hh < kG; ++hh) {
        float tm = mc[hh][0];
#pragma unroll
        for (int u = 1; u < kU; ++u) tm = fmaxf(tm, mc[hh][u]);
        const float nm = fmaxf(mx[hh], tm);
        if (nm == -INFINITY) continue;  // a head past ng
        const float corr = exp2f(mx[hh] - nm);  // 0 on the first batch
        ls[hh] *= corr;
        as[hh] *= corr;
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const float f = exp2f(mc[hh][u] - nm);  // 0 past the last chunk
          ls[hh] = fmaf(lc[hh][u], f, ls[hh]);
          as[hh] = fmaf(ac[hh][u], f, as[hh]);
        }
        mx[hh] = nm;
      }
    }
    // Parts to shared memory (reusing `red`: [part][head][e], max and sum in
    // columns D and D + 1), then part 0 combines them.
    __syncthreads();
#pragma unroll
    for (int hh = 0; hh < kG; ++hh) {
      red[part_id][hh][e] = as[hh];
      if (e == 0) {
        red[part_id][hh][D] = mx[hh];
        red[part_id][hh][D + 1] = ls[hh];
      }
    }
    __syncthreads();
    if (part_id == 0) {
#pragma unroll
      for (int hh = 0; hh < kG; ++hh) {
        if (hh >= ng) continue;
        float m2 = -INFINITY;
#pragma unroll
        for (int q2 = 0; q2 < kParts; ++q2) m2 = fmaxf(m2, red[q2][hh][D]);
        float l2 = 0.f, a2 = 0.f;
#pragma unroll
        for (int q2 = 0; q2 < kParts; ++q2) {
          const float mq = red[q2][hh][D];
          const float f = mq == -INFINITY ? 0.f : exp2f(mq - m2);  // a part without chunks
          l2 = fmaf(red[q2][hh][D + 1], f, l2);
          a2 = fmaf(red[q2][hh][e], f, a2);
        }
        const int h = hq0 + hh;
        const float a_dot = a2 / l2;
        const float a_mem = r_den[hh] != 0.f ? r_num[hh] / r_den[hh] : 0.f;
        const float gm = gate_sigmoid(gate[hh]);
        static_cast<T*>(p.out_t)[(size_t)(b * p.H_q + h) * D + e] =
            from_f32<T>(gm * a_mem + (1.f - gm) * a_dot);
      }
    }
  }
  if (threadIdx.x == 0) *ctr = 0u;  // ready for the next step
}

template <typename T, int D>
cudaError_t launch_dim(const DecodeProblem& p, cudaStream_t st) {
  const int g = p.H_q / p.H_kv;
  dim3 grid((p.pos + kRows) / kRows + 1, p.B * p.H_kv, (g + kG - 1) / kG);
  decode_step_kernel<T, D><<<grid, kThreads, 0, st>>>(p);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_type(const DecodeProblem& p, cudaStream_t st) {
  switch (p.d) {
    case 32: return launch_dim<T, 32>(p, st);
    case 64: return launch_dim<T, 64>(p, st);
    case 128: return launch_dim<T, 128>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int decode_splits(int S) { return (S + kRows - 1) / kRows; }
int decode_head_chunks(int g) { return (g + kG - 1) / kG; }

cudaError_t launch_decode_step(const DecodeProblem& p, cudaStream_t stream) {
  return p.bf16 ? launch_type<__nv_bfloat16>(p, stream) : launch_type<float>(p, stream);
}

}  // namespace infini
