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
// Transfer): that is done by the caller of these launchers, after them.
//
// Decode is bound by memory traffic (the buffer rows and M are read once per
// step), not by arithmetic, so it runs on CUDA cores:
//   decode_partial  grid (row chunks, B * H_kv, query-head chunks): one CTA
//                   streams up to 128 buffer rows of one KV head once for up
//                   to kG query heads of its group (one warp per row, lanes
//                   across d, coalesced row loads), keeping an online softmax
//                   per head in registers; partial (max, sum, acc[d]) to the
//                   workspace.  The CTA whose chunk holds row `pos` takes that
//                   row from k_t, v_t and writes it into the buffer.
//   decode_combine  grid (B * H_q), d threads: merges the chunks' partials,
//                   adds the retrieval from (M, z) and the gate, stores out_t.
#include "common.cuh"
#include "kernels.h"

namespace infini {

namespace {

constexpr int kRows = 128;      // buffer rows per CTA
constexpr int kDecThreads = 128;
constexpr int kWarps = kDecThreads / 32;
constexpr int kG = 4;           // query heads per CTA

// E consecutive elements of a row at `p` (this lane's share of d) as floats.
template <typename T, int E>
__device__ __forceinline__ void load_row(const T* p, float* x) {
#pragma unroll
  for (int e = 0; e < E; ++e) x[e] = to_f32<T>(p[e]);
}

template <typename T, int E>
__device__ __forceinline__ void copy_row(const T* src, T* dst) {
#pragma unroll
  for (int e = 0; e < E; ++e) dst[e] = src[e];
}

template <typename T, int D>
__global__ void __launch_bounds__(kDecThreads)
decode_partial(DecodeProblem p) {
  constexpr int E = D / 32;  // elements of d per lane
  __shared__ float qs[kG][D];
  __shared__ float red_m[kWarps][kG], red_l[kWarps][kG];
  __shared__ float red_acc[kWarps][kG][D];

  const int c = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / p.H_kv, hk = bh - b * p.H_kv;
  const int g = p.H_q / p.H_kv;
  const int hq0 = hk * g + blockIdx.z * kG;
  const int ng = min(kG, g - (int)blockIdx.z * kG);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = c * kRows, r1 = min(r0 + kRows, p.pos + 1);
  const T* q_t = static_cast<const T*>(p.q_t);
  const T* k_t = static_cast<const T*>(p.k_t) + (size_t)bh * D;
  const T* v_t = static_cast<const T*>(p.v_t) + (size_t)bh * D;
  T* kbuf = static_cast<T*>(p.k_buf) + (size_t)bh * p.S * D;
  T* vbuf = static_cast<T*>(p.v_buf) + (size_t)bh * p.S * D;

  // Queries in base-2 units: q * log2(e) / sqrt(d).
  const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;
  for (int i = threadIdx.x; i < kG * D; i += kDecThreads) {
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
  for (int j = r0 + warp; j < r1; j += kWarps) {
    const bool fresh = j == p.pos;
    const T* kr = fresh ? k_t : kbuf + (size_t)j * D;
    const T* vr = fresh ? v_t : vbuf + (size_t)j * D;
    float kx[E], vx[E];
    load_row<T, E>(kr + lane * E, kx);
    load_row<T, E>(vr + lane * E, vx);
    if (fresh && blockIdx.z == 0) {
      copy_row<T, E>(kr + lane * E, kbuf + (size_t)j * D + lane * E);
      copy_row<T, E>(vr + lane * E, vbuf + (size_t)j * D + lane * E);
    }
#pragma unroll
    for (int hh = 0; hh < kG; ++hh) {
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) s = fmaf(qr[hh][e], kx[e], s);
      s = warp_sum(s);
      const float mn = fmaxf(m[hh], s);
      const float corr = exp2f(m[hh] - mn);  // 0 on the first row (m = -inf)
      const float pj = exp2f(s - mn);
      l[hh] = l[hh] * corr + pj;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[hh][e] = fmaf(acc[hh][e], corr, pj * vx[e]);
      m[hh] = mn;
    }
  }
  // Merge the warps' partials.
#pragma unroll
  for (int hh = 0; hh < kG; ++hh) {
    if (lane == 0) {
      red_m[warp][hh] = m[hh];
      red_l[warp][hh] = l[hh];
    }
#pragma unroll
    for (int e = 0; e < E; ++e) red_acc[warp][hh][lane * E + e] = acc[hh][e];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < ng * D; i += kDecThreads) {
    const int hh = i / D, e = i - hh * D;
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) mx = fmaxf(mx, red_m[w][hh]);
    float ls = 0.f, as = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      // A warp without rows has m = -inf, l = acc = 0; mx is finite (the
      // chunk has at least one row).
      const float f = red_m[w][hh] == -INFINITY ? 0.f : exp2f(red_m[w][hh] - mx);
      ls = fmaf(red_l[w][hh], f, ls);
      as = fmaf(red_acc[w][hh][e], f, as);
    }
    float* part = p.part + ((size_t)(b * p.H_q + hq0 + hh) * p.nsplit + c) * (D + 2);
    part[2 + e] = as;
    if (e == 0) {
      part[0] = mx;
      part[1] = ls;
    }
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(D)
decode_combine(DecodeProblem p) {
  __shared__ float sq[D];
  __shared__ float red[D / 32];
  const int bh = blockIdx.x;  // b * H_q + h
  const int b = bh / p.H_q, h = bh - b * p.H_q;
  const int hk = h / (p.H_q / p.H_kv);
  const int t = threadIdx.x;
  const int nchunks = (p.pos + kRows) / kRows;  // chunks holding rows 0..pos

  // A_dot: merge the chunks' (max, sum, acc).
  const float* part = p.part + (size_t)bh * p.nsplit * (D + 2);
  float mx = -INFINITY;
  for (int c = 0; c < nchunks; ++c) mx = fmaxf(mx, part[(size_t)c * (D + 2)]);
  float ls = 0.f, as = 0.f;
  for (int c = 0; c < nchunks; ++c) {
    const float* pc = part + (size_t)c * (D + 2);
    const float f = exp2f(pc[0] - mx);
    ls = fmaf(pc[1], f, ls);
    as = fmaf(pc[2 + t], f, as);
  }
  const float a_dot = as / ls;

  // A_mem = sigma(q) M / (sigma(q) z), M [d_k x d_v] row-major per KV head.
  const T* q_t = static_cast<const T*>(p.q_t) + (size_t)bh * D;
  const float sqt = elu1(to_f32<T>(q_t[t]));
  sq[t] = sqt;
  const float* zv = p.z + (size_t)(b * p.H_kv + hk) * D;
  float dpart = warp_sum(sqt * zv[t]);
  if ((t & 31) == 0) red[t >> 5] = dpart;
  __syncthreads();
  float den = 0.f;
#pragma unroll
  for (int w = 0; w < D / 32; ++w) den += red[w];
  const float* Mh = p.M + (size_t)(b * p.H_kv + hk) * D * D;
  float num = 0.f;
#pragma unroll 8
  for (int i = 0; i < D; ++i) num = fmaf(sq[i], Mh[(size_t)i * D + t], num);
  const float a_mem = den != 0.f ? num / den : 0.f;

  const float gm = gate_sigmoid(p.beta[h]);
  T* out = static_cast<T*>(p.out_t) + (size_t)bh * D;
  out[t] = from_f32<T>(gm * a_mem + (1.f - gm) * a_dot);
}

template <typename T, int D>
cudaError_t launch_dim(const DecodeProblem& p, cudaStream_t st) {
  const int g = p.H_q / p.H_kv;
  dim3 grid1((p.pos + kRows) / kRows, p.B * p.H_kv, (g + kG - 1) / kG);
  decode_partial<T, D><<<grid1, kDecThreads, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_combine<T, D><<<p.B * p.H_q, D, 0, st>>>(p);
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

cudaError_t launch_decode_step(const DecodeProblem& p, cudaStream_t stream) {
  return p.bf16 ? launch_type<__nv_bfloat16>(p, stream) : launch_type<float>(p, stream);
}

}  // namespace infini
