// Backward of the Infini-attention forward (back-propagation through the
// segments), fp32 CUDA-core kernels for short segments (S <= 64, the pages'
// training rollout is 16 segments of 64: "Hugging Face Infini-Attention
// 再現分析", "重み減衰とロールアウト"; BPTT through the memory: "Leave No
// Context Behind" explainer, "限界").
//
// Given the gradients of a loss with respect to out, M_out and z_out, the
// chain rule through the forward's steps (see the forward kernels) gives the
// gradients with respect to q, k, v, beta, M_in and z_in:
//   bwd_segment (per segment and query head): recomputes sigma(Q), the
//     retrieval and the softmax, then
//       dA_mem = g dout, dA_dot = (1 - g) dout, dbeta += sum(dout (A_mem -
//       A_dot)) g (1 - g);
//       retrieval: dnum = dA_mem / den, dden = -rowsum(dA_mem A_mem) / den
//       (rows with den = 0 carry nothing), d sigma(Q) = dnum M^T + dden z^T,
//       dM_{s-1} += sigma(Q)^T dnum, dz_{s-1} += sigma(Q)^T dden;
//       attention: dV = P^T dA_dot, dP = dA_dot V^T, dS = P (dP - rowsum(dP P)),
//       dQ = dS K / sqrt(d) + d sigma(Q) sigma'(Q), dK = dS^T Q / sqrt(d);
//     writes dq, and per query head the attention's dK, dV and the
//     retrieval's dM_{s-1}, dz_{s-1} to the workspace.
//   bwd_scan (per KV head, segments in reverse): carries G_M = dL/dM_s and
//     G_z = dL/dz_s from (dM_out, dz_out); per segment the update's VJP
//       linear: d sigma(K) = V G_M^T + G_z, dV = sigma(K) G_M;
//       delta:  r = sigma(K) z, R = sigma(K) M / r, U = V - R,
//               dU = sigma(K) G_M, dV = dU, dN = -dU / r,
//               dr = rowsum(dU R) / r, d sigma(K) = U G_M^T + dN M^T +
//               dr z^T + G_z, G_M += sigma(K)^T dN, G_z += sigma(K)^T dr
//       (rows with r = 0 carry no retrieval term),
//     then adds the query heads' dM_{s-1}, dz_{s-1}; writes dk = d sigma(K)
//     sigma'(K) + the heads' attention dK, dv likewise, and finally dM_in,
//     dz_in.
//   bwd_dbeta: the per-(segment, head) gate partials summed in a fixed order.
// (M_{s-1}, z_{s-1}) come from the forward's fp32 state scan, run again.
// Every sum runs in a fixed order: the results are bitwise reproducible.
#include "common.cuh"
#include "kernels.h"

namespace infini {

namespace {

constexpr int kBwdThreads = 256;  // reverse scan, gate sum; one product group
constexpr int kSegThreads = 512;  // bwd_segment: two product groups
constexpr int kBwdMaxS = 64;

__device__ __forceinline__ float elu1_grad(float x) { return x > 0.f ? 1.f : expf(x); }

// C = A B over kk < K for the calling thread's block of an NR x NC output
// (NR, NC in {32, 64}): rows i = ti + 16u (u < NR/16), columns j = tj + 16v
// (v < NC/16), thread (ti, tj) = (t / 16, t % 16) of a group of 256 threads
// (t = tid % 256; a 512-thread CTA runs two products at once).
// A(i, kk) = A[i * lda + kk], or A[kk * lda + i] when TA; B(kk, j) =
// B[kk * ldb + j], or B[j * ldb + kk] when TB.  Per kk, NR/16 + NC/16 shared
// loads feed NR NC / 256 FMAs (16 for 64 x 64); a warp's loads of B touch 16
// consecutive addresses (or stride ldb = d + 1), so no bank conflicts.  Rows
// or columns past the operands' extent give values the caller does not
// store.  acc is added to.
template <int NR, int NC, bool TA, bool TB>
__device__ __forceinline__ void mm_tile(const float* __restrict__ A, int lda,
                                        const float* __restrict__ B, int ldb, int K,
                                        float (&acc)[NR / 16][NC / 16]) {
  const int ti = (threadIdx.x & 255) >> 4, tj = threadIdx.x & 15;
#pragma unroll 4
  for (int kk = 0; kk < K; ++kk) {
    float a[NR / 16], b[NC / 16];
#pragma unroll
    for (int u = 0; u < NR / 16; ++u) a[u] = TA ? A[kk * lda + ti + 16 * u] : A[(ti + 16 * u) * lda + kk];
#pragma unroll
    for (int v = 0; v < NC / 16; ++v) b[v] = TB ? B[(tj + 16 * v) * ldb + kk] : B[kk * ldb + tj + 16 * v];
#pragma unroll
    for (int u = 0; u < NR / 16; ++u)
#pragma unroll
      for (int v = 0; v < NC / 16; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
  }
}

template <int NR, int NC>
__device__ __forceinline__ void zero_tile(float (&acc)[NR / 16][NC / 16]) {
#pragma unroll
  for (int u = 0; u < NR / 16; ++u)
#pragma unroll
    for (int v = 0; v < NC / 16; ++v) acc[u][v] = 0.f;
}

// Calls f(i, j, value) for the thread's elements of an NR x NC tile result.
template <int NR, int NC, typename F>
__device__ __forceinline__ void for_tile(const float (&acc)[NR / 16][NC / 16], F&& f) {
  const int ti = (threadIdx.x & 255) >> 4, tj = threadIdx.x & 15;
#pragma unroll
  for (int u = 0; u < NR / 16; ++u)
#pragma unroll
    for (int v = 0; v < NC / 16; ++v) f(ti + 16 * u, tj + 16 * v, acc[u][v]);
}

// The 64 x 64 product with 128-bit shared loads, for K a multiple of 4 and
// leading dimensions a multiple of 4 floats: per four kk, four float4 loads
// of A and four of B feed 64 FMAs.  Thread (ti, tj) = (tid / 16, tid % 16):
// its rows are ti + 16u (A row-major: a float4 runs along kk) or 4ti + u
// (TA: a float4 runs along the rows), its columns 4tj + v (B row-major) or
// tj + 16v (TB: a float4 runs along kk).  A warp's B loads are 16 distinct
// 16-byte pieces in two wavefronts either way.
template <bool TA, bool TB>
__device__ __forceinline__ int vrow(int u) {
  return TA ? 4 * ((threadIdx.x & 255) >> 4) + u : ((threadIdx.x & 255) >> 4) + 16 * u;
}
template <bool TA, bool TB>
__device__ __forceinline__ int vcol(int v) {
  return TB ? (threadIdx.x & 15) + 16 * v : 4 * (threadIdx.x & 15) + v;
}

template <bool TA, bool TB>
__device__ __forceinline__ void mm_tile_v(const float* __restrict__ A, int lda,
                                          const float* __restrict__ B, int ldb, int K,
                                          float (&acc)[4][4]) {
  const int ti = (threadIdx.x & 255) >> 4, tj = threadIdx.x & 15;
#pragma unroll 2
  for (int k4 = 0; k4 < K; k4 += 4) {
    float a[4][4], b[4][4];  // a[u][t] = A(row u, k4 + t), b[t][v] = B(k4 + t, col v)
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      if (TA) {  // A[(k4 + x) * lda + 4ti .. + 3]: rows 4ti + u at kk = k4 + x
        const float4 f = *reinterpret_cast<const float4*>(A + (k4 + x) * lda + 4 * ti);
        a[0][x] = f.x; a[1][x] = f.y; a[2][x] = f.z; a[3][x] = f.w;
      } else {   // A[(ti + 16x) * lda + k4 .. + 3]: row ti + 16x
        const float4 f = *reinterpret_cast<const float4*>(A + (ti + 16 * x) * lda + k4);
        a[x][0] = f.x; a[x][1] = f.y; a[x][2] = f.z; a[x][3] = f.w;
      }
      if (TB) {  // B[(tj + 16x) * ldb + k4 .. + 3]: column tj + 16x
        const float4 f = *reinterpret_cast<const float4*>(B + (tj + 16 * x) * ldb + k4);
        b[0][x] = f.x; b[1][x] = f.y; b[2][x] = f.z; b[3][x] = f.w;
      } else {   // B[(k4 + x) * ldb + 4tj .. + 3]: columns 4tj + v at kk = k4 + x
        const float4 f = *reinterpret_cast<const float4*>(B + (k4 + x) * ldb + 4 * tj);
        b[x][0] = f.x; b[x][1] = f.y; b[x][2] = f.z; b[x][3] = f.w;
      }
    }
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u][t], b[t][v], acc[u][v]);
  }
}

// C = A B (NR x NC, over kk < K) handed to f(i, j, value) element by element:
// the 128-bit path where it applies (64 x 64, K % 4 == 0), else mm_tile.
// With a second pair (A2, B2) the two products are summed (same shapes).
template <int NR, int NC, bool TA, bool TB, typename F>
__device__ __forceinline__ void product(const float* __restrict__ A, int lda,
                                        const float* __restrict__ B, int ldb, int K, F&& f,
                                        const float* __restrict__ A2 = nullptr,
                                        const float* __restrict__ B2 = nullptr, int lda2 = 0,
                                        int ldb2 = 0) {
  if (NR == 64 && NC == 64 && (K & 3) == 0) {
    float acc[4][4];
    zero_tile<64, 64>(acc);
    mm_tile_v<TA, TB>(A, lda, B, ldb, K, acc);
    if (A2) mm_tile_v<TA, TB>(A2, lda2, B2, ldb2, K, acc);
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) f(vrow<TA, TB>(u), vcol<TA, TB>(v), acc[u][v]);
    return;
  }
  float acc[NR / 16][NC / 16];
  zero_tile<NR, NC>(acc);
  mm_tile<NR, NC, TA, TB>(A, lda, B, ldb, K, acc);
  if (A2) mm_tile<NR, NC, TA, TB>(A2, lda2, B2, ldb2, K, acc);
  for_tile<NR, NC>(acc, f);
}

// 16-byte pieces of a contiguous [rows][D] slice (element type T): the
// thread's pieces of the first `count` elements are loaded into registers
// first (all loads in flight together), then unpacked into a shared tile of
// row stride ld.
template <typename T, int D, int ROWS, int NT = kBwdThreads>
struct TileLoad {
  static constexpr int kVec = 16 / (int)sizeof(T);
  static constexpr int kPer = (ROWS * D / kVec + NT - 1) / NT;
  uint4 raw[kPer];
  __device__ __forceinline__ void issue(const T* __restrict__ src, int count) {
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = threadIdx.x + u * NT;
      raw[u] = e * kVec < count ? reinterpret_cast<const uint4*>(src)[e] : make_uint4(0, 0, 0, 0);
    }
  }
  __device__ __forceinline__ void store(float* dst, int ld, int count) const {
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = (threadIdx.x + u * NT) * kVec;
      if (e >= count) continue;
      const T* x = reinterpret_cast<const T*>(&raw[u]);
      const int i = e / D, c = e % D;  // kVec divides D: one row per piece
#pragma unroll
      for (int t = 0; t < kVec; ++t) dst[i * ld + c + t] = to_f32(x[t]);
    }
  }
  // dst += the piece's values (fp32 sources only)
  __device__ __forceinline__ void add(float* dst, int ld, int count) const {
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = (threadIdx.x + u * NT) * kVec;
      if (e >= count) continue;
      const float* x = reinterpret_cast<const float*>(&raw[u]);
      const int i = e / D, c = e % D;
#pragma unroll
      for (int t = 0; t < kVec; ++t) dst[i * ld + c + t] += x[t];
    }
  }
};

// Shared-memory plan of bwd_segment (floats): n x D tiles with row stride
// D + 4, n x n tiles with stride kBwdMaxS + 4 (16-byte aligned rows for the
// 128-bit loads; rows and columns are both read across lanes at most two
// wavefronts deep).
template <int D>
struct SegSmem {
  static constexpr int kLd = D + 4;
  static constexpr int kLp = kBwdMaxS + 4;
  static constexpr int kTile = kBwdMaxS * kLd;
  static constexpr int kQ = 0, kK = kQ + kTile, kV = kK + kTile, kDO = kV + kTile;
  static constexpr int kM = kDO + kTile;            // [D][D + 1]
  static constexpr int kX = kM + D * kLd;           // sigma(Q)
  static constexpr int kAm = kX + kTile;            // A_mem, then dQ
  static constexpr int kY = kAm + kTile;            // A_dot, then dnum
  static constexpr int kP = kY + kTile;             // [n][n] softmax
  static constexpr int kDS = kP + kBwdMaxS * kLp;   // [n][n] dP, then dS
  static constexpr int kZ = kDS + kBwdMaxS * kLp;   // z_{s-1}
  static constexpr int kDen = kZ + D;
  static constexpr int kDden = kDen + kBwdMaxS;
  static constexpr int kRs = kDden + kBwdMaxS;
  static constexpr int kRed = kRs + kBwdMaxS;       // block reduction
  static constexpr int kTotal = kRed + kSegThreads / 32;
};

// Thread groups: threads 0..255 (group 0) and 256..511 (group 1) run
// independent products of a phase side by side; row reductions use all 16
// warps.
template <typename T, int D>
__global__ void __launch_bounds__(kSegThreads)
bwd_segment(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
            const float* __restrict__ beta, const T* __restrict__ dout,
            const float* __restrict__ Mf, const float* __restrict__ zf,
            float* __restrict__ dq, float* __restrict__ dKa, float* __restrict__ dVa,
            float* __restrict__ dMr, float* __restrict__ dzr, float* __restrict__ dbp,
            int H_q, int H_kv, int L, int S, int T_seg) {
  using SM = SegSmem<D>;
  constexpr int ld = SM::kLd, lp = SM::kLp;
  constexpr int kWarps = kSegThreads / 32;
  extern __shared__ __align__(16) float sm[];
  float *Q = sm + SM::kQ, *K = sm + SM::kK, *V = sm + SM::kV, *dO = sm + SM::kDO;
  float *M = sm + SM::kM, *X = sm + SM::kX, *Am = sm + SM::kAm, *Y = sm + SM::kY;
  float *P = sm + SM::kP, *dS = sm + SM::kDS, *z = sm + SM::kZ, *den = sm + SM::kDen;
  float *dden = sm + SM::kDden, *rs = sm + SM::kRs, *red = sm + SM::kRed;
  const int s = blockIdx.x, bh = blockIdx.y;  // bh = b * H_q + h
  const int h = bh % H_q, b = bh / H_q;
  const int bhkv = b * H_kv + h / (H_q / H_kv);
  const int BHq = gridDim.y, BHkv = BHq / H_q * H_kv;
  const int r0 = s * S, n = min(S, L - r0);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = tid >> 8, gt = tid & 255;
  const float scale = rsqrtf((float)D);
  const float g = gate_sigmoid(beta[h]);
  const float ga = 1.f - g;
  constexpr int N = kBwdMaxS;  // tile extent of the segment's rows

  // ---- loads (rows past the segment stay out of every sum: loops run to n)
  const T* qs = q + ((size_t)bh * L + r0) * D;
  const T* ks = k + ((size_t)bhkv * L + r0) * D;
  const T* vs = v + ((size_t)bhkv * L + r0) * D;
  const T* ds = dout + ((size_t)bh * L + r0) * D;
  {
    TileLoad<T, D, kBwdMaxS, kSegThreads> lq, lk, lv, ld_o;
    TileLoad<float, D, D, kSegThreads> lm;
    lq.issue(qs, n * D);
    lk.issue(ks, n * D);
    lv.issue(vs, n * D);
    ld_o.issue(ds, n * D);
    lm.issue(Mf + ((size_t)s * BHkv + bhkv) * D * D, D * D);
    for (int c = tid; c < D; c += kSegThreads) z[c] = zf[((size_t)s * BHkv + bhkv) * D + c];
    lq.store(Q, ld, n * D);
    lk.store(K, ld, n * D);
    lv.store(V, ld, n * D);
    ld_o.store(dO, ld, n * D);
    lm.store(M, ld, D * D);
  }
  __syncthreads();
  for (int e = tid; e < n * D; e += kSegThreads) {
    const int i = e / D, c = e % D;
    X[i * ld + c] = elu1(Q[i * ld + c]);
  }
  __syncthreads();
  // den_i = sigma(q_i) . z
  for (int i = warp; i < n; i += kWarps) {
    float a = 0.f;
    for (int c = lane; c < D; c += 32) a = fmaf(X[i * ld + c], z[c], a);
    a = warp_sum(a);
    if (lane == 0) den[i] = a;
  }
  __syncthreads();
  if (grp == 0) {
    // scores, masked (key j <= row i)
    product<N, N, false, true>(Q, ld, K, ld, D, [&](int i, int j, float x) {
      if (i < n && j < n) P[i * lp + j] = j <= i ? x * scale : -INFINITY;
    });
  } else {
    // A_mem = sigma(Q) M / den (0 where den = 0)
    product<N, D, false, false>(X, ld, M, ld, D, [&](int i, int c, float x) {
      if (i < n) Am[i * ld + c] = den[i] != 0.f ? x / den[i] : 0.f;
    });
  }
  __syncthreads();
  // row softmax of the scores
  for (int i = warp; i < n; i += kWarps) {
    float m = -INFINITY;
    for (int j = lane; j < n; j += 32) m = fmaxf(m, P[i * lp + j]);
    m = warp_max(m);
    float l = 0.f;
    for (int j = lane; j < n; j += 32) {
      const float p = expf(P[i * lp + j] - m);
      P[i * lp + j] = p;
      l += p;
    }
    l = warp_sum(l);
    const float inv = 1.f / l;
    for (int j = lane; j < n; j += 32) P[i * lp + j] *= inv;
  }
  __syncthreads();
  if (grp == 0) {
    // A_dot = P V (P is 0 right of the diagonal), and the gate's partial
    // sum(dout (A_mem - A_dot))
    float part = 0.f;
    product<N, D, false, false>(P, lp, V, ld, n, [&](int i, int c, float x) {
      if (i < n) part = fmaf(dO[i * ld + c], Am[i * ld + c] - x, part);
    });
    part = warp_sum(part);
    if (lane == 0) red[warp] = part;
  } else {
    // dden_i = -sum_c g dout A_mem / den; dnum = g dout / den
    for (int i = warp - kWarps / 2; i < n; i += kWarps / 2) {
      float a = 0.f;
      for (int c = lane; c < D; c += 32) a = fmaf(dO[i * ld + c], Am[i * ld + c], a);
      a = warp_sum(a);
      if (lane == 0) dden[i] = den[i] != 0.f ? -g * a / den[i] : 0.f;
    }
    for (int e = gt; e < n * D; e += 256) {
      const int i = e / D, c = e % D;
      Y[i * ld + c] = den[i] != 0.f ? g * dO[i * ld + c] / den[i] : 0.f;
    }
  }
  __syncthreads();
  if (tid == 0) {
    float a = 0.f;
    for (int w = 0; w < kWarps / 2; ++w) a += red[w];
    dbp[(size_t)bh * T_seg + s] = a * g * (1.f - g);
  }
  if (grp == 0) {
    // Retrieval: dM_{s-1} += sigma(Q)^T dnum; dQ (retrieval part) =
    // (dnum M^T + dden z^T) sigma'(Q), into Am
    float* dMo = dMr + ((size_t)s * BHq + bh) * D * D;
    product<D, D, true, false>(X, ld, Y, ld, n, [&](int kk, int c, float x) { dMo[kk * D + c] = x; });
    product<N, D, false, true>(Y, ld, M, ld, D, [&](int i, int kk, float x) {
      if (i < n) Am[i * ld + kk] = fmaf(dden[i], z[kk], x) * elu1_grad(Q[i * ld + kk]);
    });
  } else {
    // Attention: dP = (1 - g) dout V^T (causal part only); dV = P^T dA_dot;
    // dz_{s-1} += sigma(Q)^T dden
    product<N, N, false, true>(dO, ld, V, ld, D, [&](int i, int j, float x) {
      if (i < n && j < n) dS[i * lp + j] = j <= i ? ga * x : 0.f;
    });
    float* dVo = dVa + ((size_t)bh * L + r0) * D;
    product<N, D, true, false>(P, lp, dO, ld, n, [&](int j, int c, float x) {
      if (j < n) dVo[j * D + c] = ga * x;
    });
    for (int kk = gt; kk < D; kk += 256) {
      float a = 0.f;
      for (int i = 0; i < n; ++i) a = fmaf(X[i * ld + kk], dden[i], a);
      dzr[((size_t)s * BHq + bh) * D + kk] = a;
    }
  }
  __syncthreads();
  // dS = P (dP - rowsum(dP P))
  for (int i = warp; i < n; i += kWarps) {
    float a = 0.f;
    for (int j = lane; j <= i; j += 32) a = fmaf(dS[i * lp + j], P[i * lp + j], a);
    a = warp_sum(a);
    if (lane == 0) rs[i] = a;
  }
  __syncthreads();
  for (int e = tid; e < n * n; e += kSegThreads) {
    const int i = e / n, j = e % n;
    dS[i * lp + j] = j <= i ? P[i * lp + j] * (dS[i * lp + j] - rs[i]) : 0.f;
  }
  __syncthreads();
  if (grp == 0) {
    // dq = dS K / sqrt(d) + retrieval part
    float* dqo = dq + ((size_t)bh * L + r0) * D;
    product<N, D, false, false>(dS, lp, K, ld, n, [&](int i, int c, float x) {
      if (i < n) dqo[i * D + c] = fmaf(x, scale, Am[i * ld + c]);
    });
  } else {
    // dK (attention) = dS^T Q / sqrt(d)
    float* dKo = dKa + ((size_t)bh * L + r0) * D;
    product<N, D, true, false>(dS, lp, Q, ld, n, [&](int j, int c, float x) {
      if (j < n) dKo[j * D + c] = x * scale;
    });
  }
}

// Shared-memory plan of bwd_scan (floats).
template <int D>
struct ScanBwdSmem {
  static constexpr int kLd = D + 4;
  static constexpr int kTile = kBwdMaxS * kLd;
  static constexpr int kGM = 0;                    // [D][D + 1] dL/dM_s
  static constexpr int kM = kGM + D * kLd;         // M_{s-1}
  static constexpr int kSK = kM + D * kLd;         // sigma(K)
  static constexpr int kV = kSK + kTile;
  static constexpr int kX1 = kV + kTile;           // d sigma(K)
  static constexpr int kX2 = kX1 + kTile;          // dV (= dU, delta)
  static constexpr int kX3 = kX2 + kTile;          // R, then U = V - R (delta)
  static constexpr int kX4 = kX3 + kTile;          // dN = -dU / r (delta)
  static constexpr int kX5 = kX4 + kTile;          // sigma(K)^T dN (delta)
  static constexpr int kGz = kX5 + kTile;
  static constexpr int kZ = kGz + D;
  static constexpr int kR = kZ + D;                // r_t (delta)
  static constexpr int kDr = kR + kBwdMaxS;        // dr_t (delta)
  static constexpr int kTotal = kDr + kBwdMaxS;
};

// 512 threads: two 256-thread groups run the independent products of a
// phase side by side; the next segment's K, V (and M_{s-1}) are in flight in
// registers while the current one is processed.
template <typename T, int D, bool DELTA>
__global__ void __launch_bounds__(kSegThreads)
bwd_scan(const T* __restrict__ k, const T* __restrict__ v, const float* __restrict__ Mf,
         const float* __restrict__ zf, const float* __restrict__ dM_out,
         const float* __restrict__ dz_out, const float* __restrict__ dKa,
         const float* __restrict__ dVa, const float* __restrict__ dMr,
         const float* __restrict__ dzr, float* __restrict__ dk, float* __restrict__ dv,
         float* __restrict__ dM_in, float* __restrict__ dz_in, int H_q, int H_kv, int L, int S,
         int T_seg) {
  using SM = ScanBwdSmem<D>;
  constexpr int ld = SM::kLd;
  constexpr int NT = kSegThreads, kWarps = NT / 32;
  extern __shared__ __align__(16) float sm[];
  float *GM = sm + SM::kGM, *M = sm + SM::kM, *sK = sm + SM::kSK, *V = sm + SM::kV;
  float *X1 = sm + SM::kX1, *X2 = sm + SM::kX2, *X3 = sm + SM::kX3, *X4 = sm + SM::kX4;
  float *X5 = sm + SM::kX5;
  float *Gz = sm + SM::kGz, *z = sm + SM::kZ, *r = sm + SM::kR, *dr = sm + SM::kDr;
  const int bhkv = blockIdx.x, BHkv = gridDim.x;
  const int b = bhkv / H_kv, j = bhkv % H_kv, grp = H_q / H_kv;
  const int BHq = BHkv / H_kv * H_q;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, half = tid >> 8;
  constexpr int N = kBwdMaxS;
  for (int e = tid; e < D * D; e += NT)
    GM[(e / D) * ld + e % D] = dM_out ? dM_out[(size_t)bhkv * D * D + e] : 0.f;
  for (int c = tid; c < D; c += NT) Gz[c] = dz_out ? dz_out[(size_t)bhkv * D + c] : 0.f;
  TileLoad<T, D, kBwdMaxS, NT> lk, lv;
  TileLoad<float, D, D, NT> lm;
  auto issue = [&](int s) {
    const int r0 = s * S, n = min(S, L - r0);
    lk.issue(k + ((size_t)bhkv * L + r0) * D, n * D);
    lv.issue(v + ((size_t)bhkv * L + r0) * D, n * D);
    if (DELTA) lm.issue(Mf + ((size_t)s * BHkv + bhkv) * D * D, D * D);
  };
  issue(T_seg - 1);
  for (int s = T_seg - 1; s >= 0; --s) {
    const int r0 = s * S, n = min(S, L - r0);
    lk.store(sK, ld, n * D);
    lv.store(V, ld, n * D);
    if (DELTA) {
      lm.store(M, ld, D * D);
      for (int c = tid; c < D; c += NT) z[c] = zf[((size_t)s * BHkv + bhkv) * D + c];
    }
    __syncthreads();
    if (s > 0) issue(s - 1);
    for (int e = tid; e < n * D; e += NT) {
      const int i = e / D, c = e % D;
      sK[i * ld + c] = elu1(sK[i * ld + c]);
    }
    __syncthreads();
    if (DELTA) {
      // r_t = sigma(k_t) . z_{s-1}
      for (int i = warp; i < n; i += kWarps) {
        float a = 0.f;
        for (int c = lane; c < D; c += 32) a = fmaf(sK[i * ld + c], z[c], a);
        a = warp_sum(a);
        if (lane == 0) r[i] = a;
      }
      __syncthreads();
      if (half == 0) {
        // R = sigma(K) M / r (0 where r = 0)
        product<N, D, false, false>(sK, ld, M, ld, D, [&](int i, int c, float x) {
          if (i < n) X3[i * ld + c] = r[i] != 0.f ? x / r[i] : 0.f;
        });
      } else {
        // dU = sigma(K) G_M
        product<N, D, false, false>(sK, ld, GM, ld, D, [&](int i, int c, float x) {
          if (i < n) X2[i * ld + c] = x;
        });
      }
      __syncthreads();
      // dr_t = rowsum(dU R) / r
      for (int i = warp; i < n; i += kWarps) {
        float a = 0.f;
        for (int c = lane; c < D; c += 32) a = fmaf(X2[i * ld + c], X3[i * ld + c], a);
        a = warp_sum(a);
        if (lane == 0) dr[i] = r[i] != 0.f ? a / r[i] : 0.f;
      }
      __syncthreads();
      // U = V - R (over R) and dN = -dU / r
      for (int e = tid; e < n * D; e += NT) {
        const int i = e / D, c = e % D;
        X3[i * ld + c] = V[i * ld + c] - X3[i * ld + c];
        X4[i * ld + c] = r[i] != 0.f ? -X2[i * ld + c] / r[i] : 0.f;
      }
      __syncthreads();
      if (half == 0) {
        // d sigma(K) = U G_M^T + dN M^T + dr z^T + G_z
        product<N, D, false, true>(X3, ld, GM, ld, D, [&](int i, int kk, float x) {
          if (i < n) X1[i * ld + kk] = x + fmaf(dr[i], z[kk], Gz[kk]);
        }, X4, M, ld, ld);
      } else {
        // sigma(K)^T dN (added to G_M below, once G_M has been read)
        product<D, D, true, false>(sK, ld, X4, ld, n, [&](int kk, int c, float x) { X5[kk * ld + c] = x; });
      }
      __syncthreads();
      // G_M += sigma(K)^T dN, G_z += sigma(K)^T dr
      for (int e = tid; e < D * D; e += NT) {
        const int kk = e / D, c = e % D;
        GM[kk * ld + c] += X5[kk * ld + c];
      }
      for (int kk = tid; kk < D; kk += NT) {
        float a = 0.f;
        for (int i = 0; i < n; ++i) a = fmaf(sK[i * ld + kk], dr[i], a);
        Gz[kk] += a;
      }
    } else {
      if (half == 0) {
        // d sigma(K) = V G_M^T + G_z
        product<N, D, false, true>(V, ld, GM, ld, D, [&](int i, int c, float x) {
          if (i < n) X1[i * ld + c] = x + Gz[c];
        });
      } else {
        // dV = sigma(K) G_M
        product<N, D, false, false>(sK, ld, GM, ld, D, [&](int i, int c, float x) {
          if (i < n) X2[i * ld + c] = x;
        });
      }
    }
    __syncthreads();
    // dk, dv of the segment: the update's part (dk through sigma'(k) = 1 or
    // e^k = sigma(k)) plus every query head's attention part, added in head
    // order; and the heads' retrieval gradients with respect to M_{s-1}.
    for (int e = tid; e < n * D; e += NT) {
      const int i = e / D, c = e % D;
      const float sk = sK[i * ld + c];
      X1[i * ld + c] *= sk > 1.f ? 1.f : sk;
    }
    __syncthreads();
    for (int hh = 0; hh < grp; ++hh) {
      const size_t head = (size_t)(b * H_q + j * grp + hh);
      TileLoad<float, D, kBwdMaxS, NT> la, lb;
      TileLoad<float, D, D, NT> lr;
      la.issue(dKa + (head * L + r0) * D, n * D);
      lb.issue(dVa + (head * L + r0) * D, n * D);
      lr.issue(dMr + ((size_t)s * BHq + head) * D * D, D * D);
      la.add(X1, ld, n * D);
      lb.add(X2, ld, n * D);
      lr.add(GM, ld, D * D);
    }
    __syncthreads();
    for (int e = tid; e < n * D; e += NT) {
      const int i = e / D, c = e % D;
      const size_t o = ((size_t)bhkv * L + r0 + i) * D + c;
      dk[o] = X1[i * ld + c];
      dv[o] = X2[i * ld + c];
    }
    for (int c = tid; c < D; c += NT) {
      float a = 0.f;
      for (int hh = 0; hh < grp; ++hh) a += dzr[((size_t)s * BHq + b * H_q + j * grp + hh) * D + c];
      Gz[c] += a;
    }
    __syncthreads();
  }
  for (int e = tid; e < D * D; e += NT)
    dM_in[(size_t)bhkv * D * D + e] = GM[(e / D) * ld + e % D];
  for (int c = tid; c < D; c += NT) dz_in[(size_t)bhkv * D + c] = Gz[c];
}

// dbeta[h] = sum over batch rows and segments of the partials, in order.
__global__ void __launch_bounds__(kBwdThreads)
bwd_dbeta(const float* __restrict__ dbp, float* __restrict__ dbeta, int B, int H_q, int T_seg) {
  for (int h = threadIdx.x; h < H_q; h += blockDim.x) {
    float a = 0.f;
    for (int b = 0; b < B; ++b)
      for (int s = 0; s < T_seg; ++s) a += dbp[((size_t)b * H_q + h) * T_seg + s];
    dbeta[h] = a;
  }
}

template <typename T, int D>
cudaError_t launch_bwd(const BackwardProblem& p, cudaStream_t st) {
  const int BHq = p.B * p.H_q, BHkv = p.B * p.H_kv;
  const size_t seg_smem = SegSmem<D>::kTotal * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(bwd_segment<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)seg_smem);
  if (e != cudaSuccess) return e;
  bwd_segment<T, D><<<dim3(p.T, BHq), kSegThreads, seg_smem, st>>>(
      static_cast<const T*>(p.q), static_cast<const T*>(p.k), static_cast<const T*>(p.v), p.beta,
      static_cast<const T*>(p.dout), p.Mf, p.zf, p.dq, p.dKa, p.dVa, p.dMr, p.dzr, p.dbp, p.H_q,
      p.H_kv, p.L, p.S, p.T);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t scan_smem = ScanBwdSmem<D>::kTotal * sizeof(float);
  auto scan = p.delta ? bwd_scan<T, D, true> : bwd_scan<T, D, false>;
  if ((e = cudaFuncSetAttribute(scan, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)scan_smem)) !=
      cudaSuccess)
    return e;
  scan<<<BHkv, kSegThreads, scan_smem, st>>>(
      static_cast<const T*>(p.k), static_cast<const T*>(p.v), p.Mf, p.zf, p.dM_out, p.dz_out, p.dKa,
      p.dVa, p.dMr, p.dzr, p.dk, p.dv, p.dM_in, p.dz_in, p.H_q, p.H_kv, p.L, p.S, p.T);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_dbeta<<<1, kBwdThreads, 0, st>>>(p.dbp, p.dbeta, p.B, p.H_q, p.T);
  return cudaGetLastError();
}

}  // namespace

bool backward_supported(int d_k, int d_v, int S) {
  return d_k == d_v && (d_k == 32 || d_k == 64) && S >= 1 && S <= kBwdMaxS;
}

cudaError_t launch_backward(const BackwardProblem& p, cudaStream_t stream) {
  if (p.d == 32) return p.bf16 ? launch_bwd<__nv_bfloat16, 32>(p, stream) : launch_bwd<float, 32>(p, stream);
  if (p.d == 64) return p.bf16 ? launch_bwd<__nv_bfloat16, 64>(p, stream) : launch_bwd<float, 64>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace infini
