// C ABI of libinfini_attn.so: argument checks, workspace layout, kernel
// dispatch.  The operation and every entry point are documented in
// include/infini_attn.h.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "infini_attn.h"
#include "common.cuh"
#include "kernels.h"

namespace infini {

// Device status word: kernels OR in a bit when a bounded wait runs out.
__device__ unsigned int g_status;

namespace {

constexpr size_t kAlign = 256;
constexpr size_t kHeader = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

bool head_dim_ok(int d) { return d == 32 || d == 64 || d == 128; }

struct Shape {
  int B, H_q, H_kv, L, d_k, d_v, S, T;
  bool bf16, delta;
  size_t elem;
  size_t q_bytes, k_bytes, v_bytes, out_bytes, beta_bytes, M_bytes, z_bytes;
  int path;
  int launches;
  // workspace layout
  size_t ws_zpref, ws_mpref, ws_g, ws_b, ws_dz, ws_total;
};

int check_shape(const infini_dims_t* d, int seg_len, int rule, Shape* s) {
  if (!d || !s) return INFINI_ERR_ARG;
  if (d->B < 1 || d->H_q < 1 || d->H_kv < 1 || d->L < 1 || seg_len < 1) return INFINI_ERR_ARG;
  if (d->H_q % d->H_kv != 0) return INFINI_ERR_ARG;
  if (rule != INFINI_RULE_LINEAR && rule != INFINI_RULE_DELTA) return INFINI_ERR_ARG;
  if (d->dtype != INFINI_DTYPE_BF16 && d->dtype != INFINI_DTYPE_F32) return INFINI_ERR_ARG;
  if (!head_dim_ok(d->d_k) || !head_dim_ok(d->d_v)) return INFINI_ERR_UNSUPPORTED;
  // Grid limits: (b, head) pairs index gridDim.y.
  if ((long long)d->B * d->H_q > 65535) return INFINI_ERR_UNSUPPORTED;
  s->B = d->B; s->H_q = d->H_q; s->H_kv = d->H_kv; s->L = d->L;
  s->d_k = d->d_k; s->d_v = d->d_v;
  s->S = seg_len;  // the last segment is simply shorter
  s->T = (int)(((long long)d->L + seg_len - 1) / seg_len);
  s->bf16 = d->dtype == INFINI_DTYPE_BF16;
  s->delta = rule == INFINI_RULE_DELTA;
  s->elem = s->bf16 ? 2 : 4;
  const size_t BHq = (size_t)d->B * d->H_q, BHkv = (size_t)d->B * d->H_kv;
  s->q_bytes = BHq * d->L * d->d_k * s->elem;
  s->k_bytes = BHkv * d->L * d->d_k * s->elem;
  s->v_bytes = BHkv * d->L * d->d_v * s->elem;
  s->out_bytes = BHq * d->L * d->d_v * s->elem;
  s->beta_bytes = (size_t)d->H_q * 4;
  s->M_bytes = BHkv * d->d_k * d->d_v * 4;
  s->z_bytes = BHkv * d->d_k * 4;
  const bool tc = tc_attention_supported(d->d_k, d->d_v, seg_len, s->bf16) &&
                  tc_scan_supported(d->d_k, d->d_v, s->bf16);
  s->path = tc ? INFINI_PATH_TCGEN05 : INFINI_PATH_SIMT;
  s->launches = tc ? 1 + tc_scan_launches(s->delta) : 2;
  const size_t mpref_elem = tc ? 2 : 4;
  s->ws_zpref = kHeader;
  s->ws_mpref = align_up(s->ws_zpref + (size_t)s->T * BHkv * d->d_k * 4);
  size_t end = align_up(s->ws_mpref + (size_t)s->T * BHkv * d->d_k * d->d_v * mpref_elem);
  s->ws_g = s->ws_b = s->ws_dz = end;
  if (tc) {
    size_t g = 0, b = 0, z = 0;
    tc_scan_workspace(d->B, d->H_kv, s->T, d->d_k, s->delta, &g, &b, &z);
    s->ws_g = end;
    s->ws_b = align_up(s->ws_g + g);
    s->ws_dz = align_up(s->ws_b + b);
    end = align_up(s->ws_dz + z);
  }
  s->ws_total = end;
  return INFINI_OK;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

struct Range {
  uintptr_t lo, hi;
};
bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }
Range rng(const void* p, size_t n) { return Range{(uintptr_t)p, (uintptr_t)p + n}; }

// Optional per-kernel event timing (benchmarks only).
constexpr int kKinds = 2;  // 0 = state scan, 1 = attention
struct TimedLaunch {
  int kind;
  cudaEvent_t a, b;
};
std::mutex g_timing_mu;
bool g_timing = false;
std::vector<TimedLaunch> g_pending;
std::vector<cudaEvent_t> g_event_pool;
double g_ms[kKinds];
int g_launches[kKinds];

cudaEvent_t pooled_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Runs `launch` on `st`, bracketed by events when timing is enabled.
template <typename F>
cudaError_t timed(int kind, cudaStream_t st, F&& launch) {
  std::unique_lock<std::mutex> lock(g_timing_mu);
  if (!g_timing) {
    lock.unlock();
    return launch();
  }
  cudaEvent_t a = pooled_event(), b = pooled_event();
  if (!a || !b) return cudaErrorMemoryAllocation;
  cudaError_t e = cudaEventRecord(a, st);
  if (e == cudaSuccess) e = launch();
  if (e == cudaSuccess) e = cudaEventRecord(b, st);
  if (e == cudaSuccess) {
    g_pending.push_back({kind, a, b});
  } else {
    g_event_pool.push_back(a);
    g_event_pool.push_back(b);
  }
  return e;
}

unsigned int* status_ptr() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
  return static_cast<unsigned int*>(p);
}

// Slot 0 of z_pref (z_in, read by segment 0): copied in for the SIMT scan;
// the tensor-core scan writes it itself (one operation less per forward).
cudaError_t seed_z(const Shape& s, const Problem& p, cudaStream_t st) {
  if (s.path == INFINI_PATH_TCGEN05) return cudaSuccess;
  return cudaMemcpyAsync(p.z_pref, p.z_in, s.z_bytes, cudaMemcpyDeviceToDevice, st);
}

// The state scan of the path `s` takes.
cudaError_t launch_state_scan(const Shape& s, const Problem& p, cudaStream_t st) {
  if (s.path != INFINI_PATH_TCGEN05) return launch_simt_state_scan(p, st);
  return launch_tc_state_scan(p, st);
}

// The forward's state scan alone over (k, v) of shape `s`: (M_in, z_in) ->
// (M_out, z_out), per-segment states in the workspace `ws` (laid out by
// check_shape).
cudaError_t run_state_scan(const Shape& s, const void* k, const void* v, const float* M_in,
                           const float* z_in, float* M_out, float* z_out, char* ws,
                           unsigned int* status, cudaStream_t st) {
  Problem p;
  p.q = nullptr; p.k = k; p.v = v; p.beta = nullptr; p.M_in = M_in; p.z_in = z_in;
  p.out = nullptr; p.M_out = M_out; p.z_out = z_out;
  p.B = s.B; p.H_q = s.H_q; p.H_kv = s.H_kv; p.L = s.L; p.d_k = s.d_k; p.d_v = s.d_v;
  p.S = s.S; p.T = s.T; p.bf16 = s.bf16; p.delta = s.delta;
  p.z_pref = reinterpret_cast<float*>(ws + s.ws_zpref);
  p.M_pref = ws + s.ws_mpref;
  p.M_pref_bf16 = s.path == INFINI_PATH_TCGEN05;
  p.Gbuf = reinterpret_cast<float*>(ws + s.ws_g);
  p.Bbuf = reinterpret_cast<float*>(ws + s.ws_b);
  p.dz = reinterpret_cast<float*>(ws + s.ws_dz);
  p.status = status;
  cudaError_t e = seed_z(s, p, st);
  if (e == cudaSuccess) e = timed(0, st, [&] { return launch_state_scan(s, p, st); });
  return e;
}

// out[i] = base[i] + parts[0][i] + ... + parts[n - 1][i] over the packed
// state [M | z]; each element summed in fp32 in part order.  (base and out
// may be the same array: each element is read before it is written by the
// same thread.)
__global__ void __launch_bounds__(256) state_sum_kernel(const float* M_base, const float* z_base,
                                                        const float* __restrict__ parts, int n_parts,
                                                        size_t nM, size_t nz, float* M_out,
                                                        float* z_out) {
  const size_t n = nM + nz;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    float acc = i < nM ? M_base[i] : z_base[i - nM];
    for (int p = 0; p < n_parts; ++p) acc += parts[(size_t)p * n + i];
    if (i < nM)
      M_out[i] = acc;
    else
      z_out[i - nM] = acc;
  }
}

}  // namespace

unsigned int* device_status_word() { return status_ptr(); }

}  // namespace infini

using namespace infini;

extern "C" {

int infini_attn_version(void) { return (1 << 16) | 0; }

const char* infini_attn_status_string(int status) {
  switch (status) {
    case INFINI_OK: return "ok";
    case INFINI_ERR_ARG: return "invalid argument (NULL pointer, size < 1, bad enum, H_q % H_kv != 0)";
    case INFINI_ERR_UNSUPPORTED: return "unsupported shape (head dims must be 32, 64 or 128; B*H_q <= 65535)";
    case INFINI_ERR_ALIAS: return "an output overlaps an input, another output or the workspace";
    case INFINI_ERR_CUDA: return "a CUDA runtime call failed";
    case INFINI_ERR_TIMEOUT: return "a kernel gave up a bounded wait (device status word set)";
    case INFINI_ERR_WORKSPACE: return "workspace too small or not 256-byte aligned";
    case INFINI_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case INFINI_ERR_SCRATCH_LIMIT:
      return "problem needs more scratch than the no-allocation entry point's static array "
             "holds; use infini_attn_forward with a workspace";
    default: return "unknown status";
  }
}

int infini_attn_init_state(float* M, float* z, int B, int H_kv, int d_k, int d_v, void* stream) {
  if (!M || !z || B < 1 || H_kv < 1 || d_k < 1 || d_v < 1) return INFINI_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t nM = (size_t)B * H_kv * d_k * d_v * sizeof(float);
  const size_t nz = (size_t)B * H_kv * d_k * sizeof(float);
  if (cudaMemsetAsync(M, 0, nM, st) != cudaSuccess) return INFINI_ERR_CUDA;
  if (cudaMemsetAsync(z, 0, nz, st) != cudaSuccess) return INFINI_ERR_CUDA;
  return INFINI_OK;
}

size_t infini_attn_workspace_bytes(const infini_dims_t* dims, int seg_len, int rule) {
  Shape s;
  if (check_shape(dims, seg_len, rule, &s) != INFINI_OK) return 0;
  return s.ws_total;
}

int infini_attn_plan(const infini_dims_t* dims, int seg_len, int rule, infini_plan_t* plan) {
  Shape s;
  int rc = check_shape(dims, seg_len, rule, &s);
  if (rc != INFINI_OK) return rc;
  if (!plan) return INFINI_ERR_ARG;
  plan->path = s.path;
  plan->launches = s.launches;
  plan->num_segments = s.T;
  plan->workspace_bytes = s.ws_total;
  return INFINI_OK;
}

int infini_attn_forward(const void* q, const void* k, const void* v, const float* beta,
                        const float* M_in, const float* z_in, int seg_len, int rule,
                        const infini_dims_t* dims, void* out, float* M_out, float* z_out,
                        void* workspace, size_t workspace_bytes, void* stream) {
  Shape s;
  int rc = check_shape(dims, seg_len, rule, &s);
  if (rc != INFINI_OK) return rc;
  if (!q || !k || !v || !beta || !M_in || !z_in || !out || !M_out || !z_out) return INFINI_ERR_ARG;
  const void* ptrs[] = {q, k, v, beta, M_in, z_in, out, M_out, z_out};
  for (const void* p : ptrs)
    if (!aligned16(p)) return INFINI_ERR_ALIGN;
  if (workspace == nullptr && workspace_bytes != 0) return INFINI_ERR_ARG;
  if (workspace != nullptr) {
    if (workspace_bytes < s.ws_total || ((uintptr_t)workspace & (kAlign - 1)) != 0)
      return INFINI_ERR_WORKSPACE;
  }
  // Aliasing: outputs may not overlap inputs or each other, except the
  // in-place state (M_out == M_in, z_out == z_in exactly).
  const Range r_out = rng(out, s.out_bytes), r_M = rng(M_out, s.M_bytes), r_z = rng(z_out, s.z_bytes);
  const Range ins[] = {rng(q, s.q_bytes), rng(k, s.k_bytes), rng(v, s.v_bytes),
                       rng(beta, s.beta_bytes), rng(M_in, s.M_bytes), rng(z_in, s.z_bytes)};
  for (int i = 0; i < 6; ++i) {
    if (overlap(r_out, ins[i])) return INFINI_ERR_ALIAS;
    if (overlap(r_M, ins[i]) && !(i == 4 && M_out == M_in)) return INFINI_ERR_ALIAS;
    if (overlap(r_z, ins[i]) && !(i == 5 && z_out == z_in)) return INFINI_ERR_ALIAS;
  }
  if (overlap(r_out, r_M) || overlap(r_out, r_z) || overlap(r_M, r_z)) return INFINI_ERR_ALIAS;
  if (workspace) {
    const Range r_ws = rng(workspace, s.ws_total);
    if (overlap(r_ws, r_out) || overlap(r_ws, r_M) || overlap(r_ws, r_z)) return INFINI_ERR_ALIAS;
    for (int i = 0; i < 6; ++i)
      if (overlap(r_ws, ins[i])) return INFINI_ERR_ALIAS;
  }

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned int* status = status_ptr();
  if (!status) return INFINI_ERR_CUDA;
  char* ws = static_cast<char*>(workspace);
  bool owned = false;
  if (!ws) {
    if (cudaMallocAsync(reinterpret_cast<void**>(&ws), s.ws_total, st) != cudaSuccess)
      return INFINI_ERR_CUDA;
    owned = true;
  }
  Problem p;
  p.q = q; p.k = k; p.v = v; p.beta = beta; p.M_in = M_in; p.z_in = z_in;
  p.out = out; p.M_out = M_out; p.z_out = z_out;
  p.B = s.B; p.H_q = s.H_q; p.H_kv = s.H_kv; p.L = s.L; p.d_k = s.d_k; p.d_v = s.d_v;
  p.S = s.S; p.T = s.T; p.bf16 = s.bf16; p.delta = s.delta;
  p.z_pref = reinterpret_cast<float*>(ws + s.ws_zpref);
  p.M_pref = ws + s.ws_mpref;
  p.M_pref_bf16 = s.path == INFINI_PATH_TCGEN05;
  p.Gbuf = reinterpret_cast<float*>(ws + s.ws_g);
  p.Bbuf = reinterpret_cast<float*>(ws + s.ws_b);
  p.dz = reinterpret_cast<float*>(ws + s.ws_dz);
  p.status = status;

  cudaError_t e = seed_z(s, p, st);
  if (e == cudaSuccess) e = timed(0, st, [&] { return launch_state_scan(s, p, st); });
  if (e == cudaSuccess)
    e = timed(1, st, [&] {
      return s.path == INFINI_PATH_TCGEN05 ? launch_tc_attention(p, st) : launch_simt_attention(p, st);
    });
  if (owned) {
    cudaError_t f = cudaFreeAsync(ws, st);
    if (e == cudaSuccess) e = f;
  }
  return e == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

int infini_attn_state_update(const void* k, const void* v, const float* M_in, const float* z_in,
                             int seg_len, int rule, const infini_dims_t* dims, float* M_out,
                             float* z_out, void* workspace, size_t workspace_bytes, void* stream) {
  Shape s;
  int rc = check_shape(dims, seg_len, rule, &s);
  if (rc != INFINI_OK) return rc;
  if (!k || !v || !M_in || !z_in || !M_out || !z_out) return INFINI_ERR_ARG;
  const void* ptrs[] = {k, v, M_in, z_in, M_out, z_out};
  for (const void* p : ptrs)
    if (!aligned16(p)) return INFINI_ERR_ALIGN;
  if (workspace == nullptr && workspace_bytes != 0) return INFINI_ERR_ARG;
  if (workspace != nullptr) {
    if (workspace_bytes < s.ws_total || ((uintptr_t)workspace & (kAlign - 1)) != 0)
      return INFINI_ERR_WORKSPACE;
  }
  const Range r_M = rng(M_out, s.M_bytes), r_z = rng(z_out, s.z_bytes);
  const Range ins[] = {rng(k, s.k_bytes), rng(v, s.v_bytes), rng(M_in, s.M_bytes), rng(z_in, s.z_bytes)};
  for (int i = 0; i < 4; ++i) {
    if (overlap(r_M, ins[i]) && !(i == 2 && M_out == M_in)) return INFINI_ERR_ALIAS;
    if (overlap(r_z, ins[i]) && !(i == 3 && z_out == z_in)) return INFINI_ERR_ALIAS;
  }
  if (overlap(r_M, r_z)) return INFINI_ERR_ALIAS;
  if (workspace) {
    const Range r_ws = rng(workspace, s.ws_total);
    if (overlap(r_ws, r_M) || overlap(r_ws, r_z)) return INFINI_ERR_ALIAS;
    for (int i = 0; i < 4; ++i)
      if (overlap(r_ws, ins[i])) return INFINI_ERR_ALIAS;
  }

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned int* status = status_ptr();
  if (!status) return INFINI_ERR_CUDA;
  char* ws = static_cast<char*>(workspace);
  bool owned = false;
  if (!ws) {
    if (cudaMallocAsync(reinterpret_cast<void**>(&ws), s.ws_total, st) != cudaSuccess)
      return INFINI_ERR_CUDA;
    owned = true;
  }
  // The scan of infini_attn_forward alone: it reads k, v and the state, and
  // writes the per-segment states to the workspace and (M_out, z_out).
  cudaError_t e = run_state_scan(s, k, v, M_in, z_in, M_out, z_out, ws, status, st);
  if (owned) {
    cudaError_t f = cudaFreeAsync(ws, st);
    if (e == cudaSuccess) e = f;
  }
  return e == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

int infini_attn_state_sum(const float* M_base, const float* z_base, const float* parts, int n_parts,
                          int B, int H_kv, int d_k, int d_v, float* M_out, float* z_out,
                          void* stream) {
  if (!M_base || !z_base || !M_out || !z_out || n_parts < 0 || (n_parts > 0 && !parts))
    return INFINI_ERR_ARG;
  if (B < 1 || H_kv < 1 || d_k < 1 || d_v < 1) return INFINI_ERR_ARG;
  const void* ptrs[] = {M_base, z_base, M_out, z_out, parts};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return INFINI_ERR_ALIGN;
  const size_t nM = (size_t)B * H_kv * d_k * d_v, nz = (size_t)B * H_kv * d_k;
  const Range r_M = rng(M_out, nM * 4), r_z = rng(z_out, nz * 4);
  const Range r_bM = rng(M_base, nM * 4), r_bz = rng(z_base, nz * 4);
  if (overlap(r_M, r_z)) return INFINI_ERR_ALIAS;
  if (overlap(r_M, r_bM) && M_out != M_base) return INFINI_ERR_ALIAS;
  if (overlap(r_z, r_bz) && z_out != z_base) return INFINI_ERR_ALIAS;
  if (overlap(r_M, r_bz) || overlap(r_z, r_bM)) return INFINI_ERR_ALIAS;
  if (n_parts > 0) {
    const Range r_p = rng(parts, (size_t)n_parts * (nM + nz) * 4);
    if (overlap(r_p, r_M) || overlap(r_p, r_z)) return INFINI_ERR_ALIAS;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t n = nM + nz;
  const size_t blocks = (n + 255) / 256;
  const unsigned grid = (unsigned)(blocks < 4096 ? blocks : 4096);
  state_sum_kernel<<<grid, 256, 0, st>>>(M_base, z_base, parts, n_parts, nM, nz, M_out, z_out);
  return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

namespace {

// Shape of the segment update a decode step runs when the segment fills: a
// forward over one segment (L = S).  Also checks the decode arguments.
// Decode workspace: [tickets | attention partials | retrieval | scan].
struct DecodeLayout {
  size_t ctr, part, ret, scan, total;
};

int decode_shape(const infini_dims_t* dims, int seg_len, int rule, Shape* s, DecodeLayout* lay) {
  if (!dims) return INFINI_ERR_ARG;
  infini_dims_t one = *dims;
  one.L = seg_len;
  int rc = check_shape(&one, seg_len, rule, s);
  if (rc != INFINI_OK) return rc;
  if (dims->d_k != dims->d_v) return INFINI_ERR_UNSUPPORTED;
  const size_t BHq = (size_t)dims->B * dims->H_q, d = dims->d_k;
  lay->ctr = 0;
  lay->part = align_up((size_t)dims->B * dims->H_kv * decode_head_chunks(dims->H_q / dims->H_kv) * 4);
  lay->ret = align_up(lay->part + BHq * decode_splits(seg_len) * (d + 2) * 4);
  lay->scan = align_up(lay->ret + BHq * (d + 1) * 4);
  lay->total = lay->scan + s->ws_total;
  return INFINI_OK;
}

}  // namespace

size_t infini_attn_decode_workspace_bytes(const infini_dims_t* dims, int seg_len, int rule) {
  Shape s;
  DecodeLayout lay;
  if (decode_shape(dims, seg_len, rule, &s, &lay) != INFINI_OK) return 0;
  return lay.total;
}

int infini_attn_decode_step(const void* q_t, const void* k_t, const void* v_t, const float* beta,
                            void* k_buf, void* v_buf, int pos, float* M, float* z, int seg_len,
                            int rule, const infini_dims_t* dims, void* out_t, void* workspace,
                            size_t workspace_bytes, void* stream) {
  Shape s;
  DecodeLayout lay;
  int rc = decode_shape(dims, seg_len, rule, &s, &lay);
  if (rc != INFINI_OK) return rc;
  if (pos < 0 || pos >= seg_len) return INFINI_ERR_ARG;
  if (!q_t || !k_t || !v_t || !beta || !k_buf || !v_buf || !M || !z || !out_t) return INFINI_ERR_ARG;
  const void* ptrs[] = {q_t, k_t, v_t, beta, k_buf, v_buf, M, z, out_t};
  for (const void* p : ptrs)
    if (!aligned16(p)) return INFINI_ERR_ALIGN;
  const size_t total = lay.total;
  if (workspace == nullptr && workspace_bytes != 0) return INFINI_ERR_ARG;
  if (workspace != nullptr) {
    if (workspace_bytes < total || ((uintptr_t)workspace & (kAlign - 1)) != 0) return INFINI_ERR_WORKSPACE;
  }
  // Per-step sizes: one token of q, k, v, out; the buffers hold S rows.
  const size_t tok_q = (size_t)s.B * s.H_q * s.d_k * s.elem, tok_kv = (size_t)s.B * s.H_kv * s.d_k * s.elem;
  const Range r_kb = rng(k_buf, s.k_bytes), r_vb = rng(v_buf, s.v_bytes), r_out = rng(out_t, tok_q);
  const Range r_M = rng(M, s.M_bytes), r_z = rng(z, s.z_bytes);
  const Range all[] = {rng(q_t, tok_q), rng(k_t, tok_kv), rng(v_t, tok_kv), rng(beta, s.beta_bytes),
                       r_kb, r_vb, r_M, r_z, r_out};
  for (int i = 0; i < 9; ++i)
    for (int j = i + 1; j < 9; ++j)
      if (j >= 4 && overlap(all[i], all[j])) return INFINI_ERR_ALIAS;  // j is written
  if (workspace) {
    const Range r_ws = rng(workspace, total);
    for (int i = 0; i < 9; ++i)
      if (overlap(r_ws, all[i])) return INFINI_ERR_ALIAS;
  }

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned int* status = status_ptr();
  if (!status) return INFINI_ERR_CUDA;
  char* ws = static_cast<char*>(workspace);
  bool owned = false;
  if (!ws) {
    if (cudaMallocAsync(reinterpret_cast<void**>(&ws), total, st) != cudaSuccess) return INFINI_ERR_CUDA;
    owned = true;
    if (cudaMemsetAsync(ws + lay.ctr, 0, lay.part - lay.ctr, st) != cudaSuccess) {
      cudaFreeAsync(ws, st);
      return INFINI_ERR_CUDA;
    }
  }
  DecodeProblem dp;
  dp.q_t = q_t; dp.k_t = k_t; dp.v_t = v_t; dp.beta = beta;
  dp.k_buf = k_buf; dp.v_buf = v_buf; dp.M = M; dp.z = z; dp.out_t = out_t;
  dp.part = reinterpret_cast<float*>(ws + lay.part);
  dp.ret = reinterpret_cast<float*>(ws + lay.ret);
  dp.ctr = reinterpret_cast<unsigned int*>(ws + lay.ctr);
  dp.B = s.B; dp.H_q = s.H_q; dp.H_kv = s.H_kv; dp.d = s.d_k; dp.S = seg_len; dp.pos = pos;
  dp.nsplit = decode_splits(seg_len);
  dp.bf16 = s.bf16;
  cudaError_t e = timed(1, st, [&] { return launch_decode_step(dp, st); });
  // The token filled the segment: M_s, z_s from the whole buffer, in place
  // (after the output above, which read M_{s-1}, z_{s-1}).
  if (e == cudaSuccess && pos == seg_len - 1)
    e = run_state_scan(s, k_buf, v_buf, M, z, M, z, ws + lay.scan, status, st);
  if (owned) {
    cudaError_t f = cudaFreeAsync(ws, st);
    if (e == cudaSuccess) e = f;
  }
  return e == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

namespace {

// Backward workspace: the forward's fp32 states (slot s = M_{s-1}, z_{s-1}),
// a scratch M_T / z_T, and the per-query-head partials.
struct BwdLayout {
  size_t zf, Mf, Mscr, zscr, dKa, dVa, dMr, dzr, dbp, g, b, dz, total;
  bool tc;  // the recompute runs the tensor-core scan (fp32 states out)
};

int backward_layout(const infini_dims_t* dims, int seg_len, int rule, Shape* s, BwdLayout* lay) {
  int rc = check_shape(dims, seg_len, rule, s);
  if (rc != INFINI_OK) return rc;
  if (!backward_supported(s->d_k, s->d_v, seg_len)) return INFINI_ERR_UNSUPPORTED;
  const size_t d = s->d_k, T = s->T, L = s->L;
  const size_t BHq = (size_t)s->B * s->H_q, BHkv = (size_t)s->B * s->H_kv;
  lay->zf = kHeader;
  lay->Mf = align_up(lay->zf + T * BHkv * d * 4);
  lay->Mscr = align_up(lay->Mf + T * BHkv * d * d * 4);
  lay->zscr = align_up(lay->Mscr + BHkv * d * d * 4);
  lay->dKa = align_up(lay->zscr + BHkv * d * 4);
  lay->dVa = align_up(lay->dKa + BHq * L * d * 4);
  lay->dMr = align_up(lay->dVa + BHq * L * d * 4);
  lay->dzr = align_up(lay->dMr + T * BHq * d * d * 4);
  lay->dbp = align_up(lay->dzr + T * BHq * d * 4);
  lay->g = lay->b = lay->dz = align_up(lay->dbp + BHq * T * 4);
  lay->tc = tc_scan_supported(s->d_k, s->d_v, s->bf16);
  size_t end = lay->g;
  if (lay->tc) {
    size_t g = 0, b = 0, z = 0;
    tc_scan_workspace(s->B, s->H_kv, s->T, s->d_k, s->delta, &g, &b, &z);
    lay->b = align_up(lay->g + g);
    lay->dz = align_up(lay->b + b);
    end = align_up(lay->dz + z);
  }
  lay->total = end;
  return INFINI_OK;
}

}  // namespace

size_t infini_attn_backward_workspace_bytes(const infini_dims_t* dims, int seg_len, int rule) {
  Shape s;
  BwdLayout lay;
  return backward_layout(dims, seg_len, rule, &s, &lay) == INFINI_OK ? lay.total : 0;
}

int infini_attn_backward(const void* q, const void* k, const void* v, const float* beta,
                         const float* M_in, const float* z_in, int seg_len, int rule,
                         const infini_dims_t* dims, const void* dout, const float* dM_out,
                         const float* dz_out, float* dq, float* dk, float* dv, float* dbeta,
                         float* dM_in, float* dz_in, void* workspace, size_t workspace_bytes,
                         void* stream) {
  Shape s;
  BwdLayout lay;
  int rc = backward_layout(dims, seg_len, rule, &s, &lay);
  if (rc != INFINI_OK) return rc;
  if (!q || !k || !v || !beta || !M_in || !z_in || !dout || !dq || !dk || !dv || !dbeta || !dM_in ||
      !dz_in)
    return INFINI_ERR_ARG;
  const void* ptrs[] = {q, k, v, beta, M_in, z_in, dout, dM_out, dz_out, dq, dk, dv, dbeta, dM_in, dz_in};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return INFINI_ERR_ALIGN;
  if (workspace == nullptr && workspace_bytes != 0) return INFINI_ERR_ARG;
  if (workspace && (workspace_bytes < lay.total || ((uintptr_t)workspace & (kAlign - 1)) != 0))
    return INFINI_ERR_WORKSPACE;
  const size_t dq_bytes = (size_t)s.B * s.H_q * s.L * s.d_k * 4;
  const size_t dkv_bytes = (size_t)s.B * s.H_kv * s.L * s.d_k * 4;
  const Range outs[] = {rng(dq, dq_bytes), rng(dk, dkv_bytes), rng(dv, dkv_bytes),
                        rng(dbeta, s.beta_bytes), rng(dM_in, s.M_bytes), rng(dz_in, s.z_bytes)};
  const Range ins[] = {rng(q, s.q_bytes), rng(k, s.k_bytes), rng(v, s.v_bytes),
                       rng(beta, s.beta_bytes), rng(M_in, s.M_bytes), rng(z_in, s.z_bytes),
                       rng(dout, s.out_bytes), rng(dM_out, dM_out ? s.M_bytes : 0),
                       rng(dz_out, dz_out ? s.z_bytes : 0)};
  for (int i = 0; i < 6; ++i) {
    for (int j = i + 1; j < 6; ++j)
      if (overlap(outs[i], outs[j])) return INFINI_ERR_ALIAS;
    for (const Range& r : ins)
      if (overlap(outs[i], r)) return INFINI_ERR_ALIAS;
    if (workspace && overlap(outs[i], rng(workspace, lay.total))) return INFINI_ERR_ALIAS;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned int* status = status_ptr();
  if (!status) return INFINI_ERR_CUDA;
  char* ws = static_cast<char*>(workspace);
  bool owned = false;
  if (!ws) {
    if (cudaMallocAsync(reinterpret_cast<void**>(&ws), lay.total, st) != cudaSuccess) return INFINI_ERR_CUDA;
    owned = true;
  }
  // The forward's states M_{s-1}, z_{s-1} in fp32: the fp32 state scan, run again.
  Problem p;
  p.q = q; p.k = k; p.v = v; p.beta = beta; p.M_in = M_in; p.z_in = z_in;
  p.out = nullptr;
  p.M_out = reinterpret_cast<float*>(ws + lay.Mscr);
  p.z_out = reinterpret_cast<float*>(ws + lay.zscr);
  p.B = s.B; p.H_q = s.H_q; p.H_kv = s.H_kv; p.L = s.L; p.d_k = s.d_k; p.d_v = s.d_v;
  p.S = s.S; p.T = s.T; p.bf16 = s.bf16; p.delta = s.delta;
  p.z_pref = reinterpret_cast<float*>(ws + lay.zf);
  p.M_pref = ws + lay.Mf;
  p.M_pref_bf16 = false;
  p.Gbuf = reinterpret_cast<float*>(ws + lay.g);
  p.Bbuf = reinterpret_cast<float*>(ws + lay.b);
  p.dz = reinterpret_cast<float*>(ws + lay.dz);
  p.status = status;
  cudaError_t e = cudaSuccess;
  if (lay.tc) {
    e = timed(0, st, [&] { return launch_tc_state_scan(p, st); });
  } else {
    e = cudaMemcpyAsync(p.z_pref, z_in, s.z_bytes, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess) e = timed(0, st, [&] { return launch_simt_state_scan(p, st); });
  }
  BackwardProblem bp;
  bp.q = q; bp.k = k; bp.v = v; bp.beta = beta; bp.dout = dout; bp.dM_out = dM_out; bp.dz_out = dz_out;
  bp.dq = dq; bp.dk = dk; bp.dv = dv; bp.dbeta = dbeta; bp.dM_in = dM_in; bp.dz_in = dz_in;
  bp.Mf = reinterpret_cast<const float*>(ws + lay.Mf);
  bp.zf = reinterpret_cast<const float*>(ws + lay.zf);
  bp.dKa = reinterpret_cast<float*>(ws + lay.dKa);
  bp.dVa = reinterpret_cast<float*>(ws + lay.dVa);
  bp.dMr = reinterpret_cast<float*>(ws + lay.dMr);
  bp.dzr = reinterpret_cast<float*>(ws + lay.dzr);
  bp.dbp = reinterpret_cast<float*>(ws + lay.dbp);
  bp.B = s.B; bp.H_q = s.H_q; bp.H_kv = s.H_kv; bp.L = s.L; bp.d = s.d_k; bp.S = s.S; bp.T = s.T;
  bp.bf16 = s.bf16; bp.delta = s.delta;
  if (e == cudaSuccess) e = timed(1, st, [&] { return launch_backward(bp, st); });
  if (owned) {
    cudaError_t f = cudaFreeAsync(ws, st);
    if (e == cudaSuccess) e = f;
  }
  return e == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

size_t infini_attn_host_arena_bytes(const infini_dims_t* dims, int seg_len, int rule) {
  Shape s;
  if (check_shape(dims, seg_len, rule, &s) != INFINI_OK) return 0;
  return align_up(s.q_bytes) + align_up(s.k_bytes) + align_up(s.v_bytes) + align_up(s.beta_bytes) +
         2 * align_up(s.M_bytes) + 2 * align_up(s.z_bytes) + align_up(s.out_bytes) + s.ws_total;
}

int infini_attn_forward_host(const void* q_h, const void* k_h, const void* v_h,
                             const float* beta_h, const float* M_in_h, const float* z_in_h,
                             int seg_len, int rule, const infini_dims_t* dims,
                             void* out_h, float* M_out_h, float* z_out_h,
                             void* arena, size_t arena_bytes, void* stream) {
  Shape s;
  int rc = check_shape(dims, seg_len, rule, &s);
  if (rc != INFINI_OK) return rc;
  if (!q_h || !k_h || !v_h || !beta_h || !M_in_h || !z_in_h || !out_h || !M_out_h || !z_out_h ||
      !arena)
    return INFINI_ERR_ARG;
  if (arena_bytes < infini_attn_host_arena_bytes(dims, seg_len, rule) ||
      ((uintptr_t)arena & (kAlign - 1)) != 0)
    return INFINI_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* a = static_cast<char*>(arena);
  size_t off = 0;
  auto take = [&](size_t n) { char* p = a + off; off += align_up(n); return p; };
  char* q = take(s.q_bytes);
  char* k = take(s.k_bytes);
  char* v = take(s.v_bytes);
  float* beta = reinterpret_cast<float*>(take(s.beta_bytes));
  float* M = reinterpret_cast<float*>(take(s.M_bytes));
  float* z = reinterpret_cast<float*>(take(s.z_bytes));
  float* M2 = reinterpret_cast<float*>(take(s.M_bytes));
  float* z2 = reinterpret_cast<float*>(take(s.z_bytes));
  char* out = take(s.out_bytes);
  char* ws = a + off;
  const struct { void* dst; const void* src; size_t n; } h2d[] = {
      {q, q_h, s.q_bytes}, {k, k_h, s.k_bytes}, {v, v_h, s.v_bytes},
      {beta, beta_h, s.beta_bytes}, {M, M_in_h, s.M_bytes}, {z, z_in_h, s.z_bytes}};
  for (const auto& c : h2d)
    if (cudaMemcpyAsync(c.dst, c.src, c.n, cudaMemcpyHostToDevice, st) != cudaSuccess)
      return INFINI_ERR_CUDA;
  rc = infini_attn_forward(q, k, v, beta, M, z, seg_len, rule, dims, out, M2, z2, ws, s.ws_total,
                           stream);
  if (rc != INFINI_OK) return rc;
  if (cudaMemcpyAsync(out_h, out, s.out_bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemcpyAsync(M_out_h, M2, s.M_bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemcpyAsync(z_out_h, z2, s.z_bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return INFINI_ERR_CUDA;
  return INFINI_OK;
}

int infini_attn_set_kernel_timing(int enable) {
  std::lock_guard<std::mutex> lock(g_timing_mu);
  g_timing = enable != 0;
  return INFINI_OK;
}

int infini_attn_kernel_times(double* ms, int* launches, int n_kinds, int reset) {
  if (!ms || !launches || n_kinds < 1) return INFINI_ERR_ARG;
  std::lock_guard<std::mutex> lock(g_timing_mu);
  for (const TimedLaunch& t : g_pending) {
    float el = 0.f;
    if (cudaEventSynchronize(t.b) != cudaSuccess) return INFINI_ERR_CUDA;
    if (cudaEventElapsedTime(&el, t.a, t.b) != cudaSuccess) return INFINI_ERR_CUDA;
    g_ms[t.kind] += el;
    g_launches[t.kind] += 1;
    g_event_pool.push_back(t.a);
    g_event_pool.push_back(t.b);
  }
  g_pending.clear();
  for (int k = 0; k < n_kinds; ++k) {
    ms[k] = k < kKinds ? g_ms[k] : 0.0;
    launches[k] = k < kKinds ? g_launches[k] : 0;
  }
  if (reset)
    for (int k = 0; k < kKinds; ++k) {
      g_ms[k] = 0.0;
      g_launches[k] = 0;
    }
  return INFINI_OK;
}

int infini_attn_qkv_project(const void* x, const void* w_qkv, const float* bias,
                            const float* rope_cos, const float* rope_sin, const infini_dims_t* dims,
                            int d_model, void* q, void* k, void* v, void* stream) {
  if (!dims || !x || !w_qkv || !q || !k || !v) return INFINI_ERR_ARG;
  if ((rope_cos == nullptr) != (rope_sin == nullptr)) return INFINI_ERR_ARG;
  if (dims->B < 1 || dims->H_q < 1 || dims->H_kv < 1 || dims->L < 1 || d_model < 1 ||
      dims->d_k < 1 || dims->d_v < 1)
    return INFINI_ERR_ARG;
  if (dims->dtype != INFINI_DTYPE_BF16 && dims->dtype != INFINI_DTYPE_F32) return INFINI_ERR_ARG;
  if (!qkv_projection_supported(dims->d_k, dims->d_v, d_model, dims->dtype == INFINI_DTYPE_BF16))
    return INFINI_ERR_UNSUPPORTED;
  const long long rows = (long long)dims->B * dims->L;
  if (rows > 0x7fffffffLL) return INFINI_ERR_UNSUPPORTED;
  const int d = dims->d_k;
  const size_t N = (size_t)(dims->H_q + 2 * dims->H_kv) * d;
  const void* ptrs[] = {x, w_qkv, bias, rope_cos, rope_sin, q, k, v};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return INFINI_ERR_ALIGN;
  const Range ins[] = {rng(x, (size_t)rows * d_model * 2), rng(w_qkv, N * d_model * 2),
                       rng(bias, bias ? N * 4 : 0), rng(rope_cos, rope_cos ? (size_t)dims->L * d / 2 * 4 : 0),
                       rng(rope_sin, rope_sin ? (size_t)dims->L * d / 2 * 4 : 0)};
  const Range outs[] = {rng(q, (size_t)rows * dims->H_q * d * 2),
                        rng(k, (size_t)rows * dims->H_kv * d * 2),
                        rng(v, (size_t)rows * dims->H_kv * d * 2)};
  for (int i = 0; i < 3; ++i) {
    for (const Range& r : ins)
      if (overlap(outs[i], r)) return INFINI_ERR_ALIAS;
    for (int j = i + 1; j < 3; ++j)
      if (overlap(outs[i], outs[j])) return INFINI_ERR_ALIAS;
  }
  unsigned int* status = status_ptr();
  if (!status) return INFINI_ERR_CUDA;
  ProjectionProblem p;
  p.x = x;
  p.w = w_qkv;
  p.bias = bias;
  p.rope_cos = rope_cos;
  p.rope_sin = rope_sin;
  p.q = q;
  p.k = k;
  p.v = v;
  p.B = dims->B;
  p.H_q = dims->H_q;
  p.H_kv = dims->H_kv;
  p.L = dims->L;
  p.d = d;
  p.d_model = d_model;
  p.status = status;
  return launch_qkv_projection(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? INFINI_OK
                                                                                    : INFINI_ERR_CUDA;
}

int infini_attn_rope_tables(float* cos_out, float* sin_out, int n_pos, int d, double base,
                            void* stream) {
  if (!cos_out || !sin_out || n_pos < 1 || d < 2 || d % 2 != 0 || !(base > 0.0))
    return INFINI_ERR_ARG;
  const size_t n = (size_t)n_pos * (d / 2) * 4;
  if (overlap(rng(cos_out, n), rng(sin_out, n))) return INFINI_ERR_ALIAS;
  return launch_rope_tables(cos_out, sin_out, n_pos, d, base, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? INFINI_OK
             : INFINI_ERR_CUDA;
}

int infini_attn_sync_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return INFINI_ERR_CUDA;
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, g_status, sizeof(word)) != cudaSuccess) return INFINI_ERR_CUDA;
  if (word != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return INFINI_ERR_CUDA;
    return (word & infini::kStatusLayout) ? INFINI_ERR_UNSUPPORTED : INFINI_ERR_TIMEOUT;
  }
  return INFINI_OK;
}

}  // extern "C"
