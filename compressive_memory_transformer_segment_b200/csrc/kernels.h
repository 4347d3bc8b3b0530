// Internal launcher declarations shared by the C-ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace infini {

// Problem description handed from the C-ABI layer to the launchers.
struct Problem {
  const void* q;
  const void* k;
  const void* v;
  const float* beta;
  const float* M_in;
  const float* z_in;   // the tensor-core scan seeds slot 0 of z_pref from it
  void* out;
  float* M_out;
  float* z_out;
  int B, H_q, H_kv, L, d_k, d_v, S, T;
  bool bf16;
  bool delta;
  // Workspace views.
  float* z_pref;       // [T][B*H_kv][d_k] f32: z_{s-1} read by segment s (slot 0 = z_in:
                       // copied in before the SIMT scan, written by the tensor-core scan)
  void* M_pref;        // [T][B*H_kv][d_k][d_v]: M_{s-1} (f32 on the SIMT path, bf16 on tcgen05)
  bool M_pref_bf16;    // element type of M_pref
  // Tensor-core scan only: per (segment, KV head) products and column sums.
  float* Gbuf;         // [T][B*H_kv][d][d] f32 (delta rule)
  float* Bbuf;         // [T][B*H_kv][d][d] f32
  float* dz;           // [T][B*H_kv][d] f32
  unsigned int* status;  // device status word
};

// fp32 CUDA-core path (any S, any supported d, f32 or bf16 I/O).
cudaError_t launch_simt_state_scan(const Problem& p, cudaStream_t stream);
cudaError_t launch_simt_attention(const Problem& p, cudaStream_t stream);

// Tensor-core (tcgen05 / TMEM / TMA) segment attention: bf16 I/O,
// d_k == d_v in {64, 128}, S a multiple of 128 (persistent kernel) or a
// divisor of 128 with (128 / S) * d <= 256 (short-segment kernel).  Reads
// bf16 M_pref.
bool tc_attention_supported(int d_k, int d_v, int S, bool bf16);
bool tc_small_attention_supported(int d_k, int d_v, int S, bool bf16);
cudaError_t launch_tc_small_attention(const Problem& p, cudaStream_t stream);
// Device address of the status word the kernels set (see common.cuh).
unsigned int* device_status_word();

cudaError_t launch_tc_attention(const Problem& p, cudaStream_t stream);
// The one-query-tile-per-CTA variant (used when H_q == H_kv).
cudaError_t launch_tc_attention_single(const Problem& p, cudaStream_t stream);

// Tensor-core memory-state scan (both rules): bf16 I/O, d_k == d_v in
// {64, 128}, any S.  Writes M_pref (bf16, or fp32 when !M_pref_bf16) and
// fp32 z_pref; needs the Gbuf, Bbuf and dz workspace regions sized by
// tc_scan_workspace.
bool tc_scan_supported(int d_k, int d_v, bool bf16);
int tc_scan_launches(bool delta);
void tc_scan_workspace(int B, int H_kv, int T, int d, bool delta, size_t* g_bytes, size_t* b_bytes,
                       size_t* dz_bytes);
cudaError_t launch_tc_state_scan(const Problem& p, cudaStream_t stream);

// Streaming decode step (one new token per head; CUDA cores): attention of
// q_t over rows 0..pos of the segment buffer (row pos taken from k_t, v_t and
// written into the buffer), retrieval from (M, z), gate -> out_t.
struct DecodeProblem {
  const void* q_t;     // [B, H_q, d]
  const void* k_t;     // [B, H_kv, d]
  const void* v_t;     // [B, H_kv, d]
  const float* beta;   // [H_q]
  void* k_buf;         // [B, H_kv, S, d]
  void* v_buf;         // [B, H_kv, S, d]
  const float* M;      // [B, H_kv, d, d] f32 (M_{s-1})
  const float* z;      // [B, H_kv, d] f32 (z_{s-1})
  void* out_t;         // [B, H_q, d]
  float* part;         // workspace: [B * H_q][nsplit][d + 2] f32 (attention partials)
  float* ret;          // workspace: [B * H_q][d + 1] f32 (sigma(q) M, sigma(q).z)
  unsigned int* ctr;   // workspace: [B * H_kv][head chunks] tickets, 0 between steps
  int B, H_q, H_kv, d, S, pos, nsplit;
  bool bf16;
};
// Backward through the segments (fp32 CUDA cores; S <= 64, d_k == d_v in
// {32, 64}).  Mf / zf hold the forward's per-segment states M_{s-1}, z_{s-1}
// in fp32 (from the SIMT state scan); the rest of the workspace holds the
// per-query-head partials that the reverse scan sums in a fixed order.
struct BackwardProblem {
  const void* q;
  const void* k;
  const void* v;
  const float* beta;
  const void* dout;     // [B, H_q, L, d] in the I/O dtype
  const float* dM_out;  // [B, H_kv, d, d] or NULL (zero)
  const float* dz_out;  // [B, H_kv, d] or NULL (zero)
  float* dq;            // [B, H_q, L, d]
  float* dk;            // [B, H_kv, L, d]
  float* dv;            // [B, H_kv, L, d]
  float* dbeta;         // [H_q]
  float* dM_in;         // [B, H_kv, d, d]
  float* dz_in;         // [B, H_kv, d]
  // workspace
  const float* Mf;      // [T][B*H_kv][d][d]
  const float* zf;      // [T][B*H_kv][d]
  float* dKa;           // [B*H_q][L][d]  attention's dK per query head
  float* dVa;           // [B*H_q][L][d]  attention's dV per query head
  float* dMr;           // [T][B*H_q][d][d]  retrieval's dM_{s-1} per query head
  float* dzr;           // [T][B*H_q][d]
  float* dbp;           // [B*H_q][T]  gate partials
  int B, H_q, H_kv, L, d, S, T;
  bool bf16, delta;
};
bool backward_supported(int d_k, int d_v, int S);
cudaError_t launch_backward(const BackwardProblem& p, cudaStream_t stream);

// Q/K/V projections with rotary embedding (tcgen05 GEMM with the bias, the
// rotation and the head split in its epilogue): bf16, d in {64, 128},
// d_model >= 64 and a multiple of 8.
struct ProjectionProblem {
  const void* x;         // [B * L][d_model] bf16
  const void* w;         // [(H_q + 2 H_kv) d][d_model] bf16
  const float* bias;     // [(H_q + 2 H_kv) d] or null
  const float* rope_cos; // [L][d / 2] or null (no rotation)
  const float* rope_sin;
  void* q;               // [B, H_q, L, d] bf16
  void* k;               // [B, H_kv, L, d]
  void* v;               // [B, H_kv, L, d]
  int B, H_q, H_kv, L, d, d_model;
  unsigned int* status;
};
bool qkv_projection_supported(int d_k, int d_v, int d_model, bool bf16);
cudaError_t launch_qkv_projection(const ProjectionProblem& p, cudaStream_t stream);
cudaError_t launch_rope_tables(float* cos_out, float* sin_out, int n_pos, int d, double base,
                               cudaStream_t stream);

int decode_splits(int S);
int decode_head_chunks(int g);
cudaError_t launch_decode_step(const DecodeProblem& p, cudaStream_t stream);

}  // namespace infini
