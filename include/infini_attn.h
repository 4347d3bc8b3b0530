/*
 * infini_attn.h -- C ABI of libinfini_attn.so, a B200 (sm_100a) implementation
 * of the Infini-attention layer forward pass.
 *
 * The operation.  For every batch row b and query head h (KV head
 * kv = floor(h / (H_q / H_kv))), the sequence of length L is cut into
 * T = ceil(L / S) segments of S rows (the last may be shorter), scanned in
 * order s = 1..T.  In segment s, with Q, K, V the segment's rows:
 *   A_dot = softmax(Q K^T / sqrt(d_k) + causal mask (key j <= query i)) V
 *   A_mem = sigma(Q) M_{s-1} / (sigma(Q) z_{s-1})  row-wise, 0 where the
 *           denominator is exactly 0; sigma(x) = ELU(x) + 1
 *   out   = sg(beta_h) A_mem + (1 - sg(beta_h)) A_dot,  sg = logistic
 * and then the KV head's memory is updated with the segment's keys/values:
 *   linear: M_s = M_{s-1} + sigma(K)^T V
 *   delta : M_s = M_{s-1} + sigma(K)^T (V - sigma(K) M_{s-1} / (sigma(K) z_{s-1}))
 *           (retrieval term 0 on rows whose denominator is 0)
 *   both  : z_s = z_{s-1} + sum over the segment's rows of sigma(K)
 * Only (M, z) pass from one segment to the next; after segment T they are
 * returned as (M_out, z_out).
 *
 * Where this is defined:
 *   "Hugging Face Infini-Attention 再現分析", section "Infini-Attention
 *   メカニズム": Segmentation, Local Attention, Memory Retrieval (ELU + 1),
 *   Integration (sigmoid of a learned per-head beta), Memory Update, State
 *   Transfer.
 *   "Leave No Context Behind" explainer, sections "メモリ構造" (one associative
 *   matrix per head, the attention's own Q/K/V), "メモリの読み出し"
 *   (normalised by the sum of past keys), "メモリの更新" (outer-product
 *   accumulation; the delta rule writes only the difference),
 *   "長期情報と短期情報の統合" (per-head gate), "実装上の流れ" (read, mix,
 *   then update with the current K/V).
 *   "Как работает Infini-attention", section 3, equation 1: the 1/sqrt(d)
 *   softmax scale.
 *
 * Conventions for every entry point below:
 *   - Device pointers point to memory of the current CUDA device; host
 *     pointers are marked as such.  The caller owns every buffer; the library
 *     keeps no pointer after a call returns.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is
 *     enqueued on it and the call returns without waiting for the GPU.
 *   - Return value: an infini_status_t (0 = success, negative = error).
 *     Argument errors are detected before anything is enqueued.
 */
#ifndef INFINI_ATTN_H
#define INFINI_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define INFINI_API __attribute__((visibility("default")))
#else
#define INFINI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  INFINI_RULE_LINEAR = 0,   /* M_s = M_{s-1} + sigma(K)^T V               */
  INFINI_RULE_DELTA = 1     /* M_s = M_{s-1} + sigma(K)^T (V - retrieved)  */
} infini_rule_t;

typedef enum {
  INFINI_DTYPE_BF16 = 0,    /* q, k, v, out in bfloat16; fp32 arithmetic   */
  INFINI_DTYPE_F32 = 1      /* q, k, v, out in float32; fp32 arithmetic    */
} infini_dtype_t;

typedef enum {
  INFINI_OK = 0,
  INFINI_ERR_ARG = -1,          /* bad size, NULL pointer, bad enum value   */
  INFINI_ERR_UNSUPPORTED = -2,  /* valid but unsupported shape (head dims)  */
  INFINI_ERR_ALIAS = -3,        /* an output overlaps an input or another output */
  INFINI_ERR_CUDA = -4,         /* a CUDA runtime call failed               */
  INFINI_ERR_TIMEOUT = -5,      /* a kernel gave up waiting (device-side)   */
  INFINI_ERR_WORKSPACE = -6,    /* workspace too small or misaligned        */
  INFINI_ERR_ALIGN = -7,        /* a pointer is not 16-byte aligned         */
  INFINI_ERR_SCRATCH_LIMIT = -8 /* problem too large for infini_attn_forward_noalloc */
} infini_status_t;

/* Problem sizes.  Layouts (all contiguous, row-major):
 *   q   [B, H_q,  L, d_k]   dtype          k [B, H_kv, L, d_k]   dtype
 *   v   [B, H_kv, L, d_v]   dtype        out [B, H_q,  L, d_v]   dtype
 *   beta[H_q] float32 (raw logit; sg is applied inside)
 *   M   [B, H_kv, d_k, d_v] float32        z [B, H_kv, d_k]      float32
 * Supported: B, H_q, H_kv, L >= 1; H_q % H_kv == 0; d_k, d_v in {32, 64, 128}.
 */
typedef struct {
  int B, H_q, H_kv, L, d_k, d_v;
  int dtype;                    /* an infini_dtype_t */
} infini_dims_t;

/* Which kernels a call will run (reported by infini_attn_plan). */
typedef enum {
  INFINI_PATH_SIMT = 0,         /* fp32 CUDA-core kernels (any S, fp32 I/O)  */
  INFINI_PATH_TCGEN05 = 1       /* tcgen05/TMEM tensor-core kernels (bf16)   */
} infini_path_t;

typedef struct {
  int path;                     /* an infini_path_t                          */
  int launches;                 /* kernels enqueued by one infini_attn_forward */
  int num_segments;             /* T = ceil(L / seg_len)                     */
  size_t workspace_bytes;       /* = infini_attn_workspace_bytes(...)        */
} infini_plan_t;

/* Library version, (major << 16) | minor. */
INFINI_API int infini_attn_version(void);

/* Static, NUL-terminated description of a status code. Never NULL. */
INFINI_API const char* infini_attn_status_string(int status);

/* Zero a memory state: M_0 = 0, z_0 = 0 (the empty memory every stream starts
 * from; "Hugging Face Infini-Attention 再現分析", Memory Update starts from an
 * empty buffer).  M: device [B, H_kv, d_k, d_v] f32; z: device [B, H_kv, d_k]
 * f32.  Enqueued on `stream`.  Errors: INFINI_ERR_ARG (NULL or sizes < 1),
 * INFINI_ERR_CUDA. */
INFINI_API int infini_attn_init_state(float* M, float* z, int B, int H_kv, int d_k, int d_v,
                           void* stream);

/* Bytes of device workspace infini_attn_forward needs for these sizes (the
 * memory read by each segment, kept for all T segments, plus a 256-byte
 * header).  0 if the arguments are invalid. */
INFINI_API size_t infini_attn_workspace_bytes(const infini_dims_t* dims, int seg_len, int rule);

/* Fill *plan for these sizes.  Returns INFINI_OK or the error that
 * infini_attn_forward would return for them (before touching the GPU). */
INFINI_API int infini_attn_plan(const infini_dims_t* dims, int seg_len, int rule, infini_plan_t* plan);

/* The layer forward (see the top of this file).
 *   q, k, v          device, layouts above, element type dims->dtype
 *   beta             device float32 [H_q]
 *   M_in, z_in       device float32 state read by the first segment
 *   seg_len          S >= 1
 *   rule             an infini_rule_t
 *   out              device [B, H_q, L, d_v], element type dims->dtype
 *   M_out, z_out     device float32 state after the last segment.  M_out may
 *                    equal M_in and z_out may equal z_in (in-place streaming:
 *                    feed the next call the state this call returns); any other
 *                    overlap between an output and an input, another output or
 *                    the workspace is INFINI_ERR_ALIAS.
 *   workspace        device scratch of `workspace_bytes` >= the size
 *                    infini_attn_workspace_bytes reports, 256-byte aligned;
 *                    or NULL with workspace_bytes == 0, in which case the call
 *                    takes it with cudaMallocAsync on `stream` and frees it
 *                    with cudaFreeAsync after the last kernel.
 *   stream           cudaStream_t.
 * All pointers must be 16-byte aligned (INFINI_ERR_ALIGN).  Device-side
 * failures (a kernel that gave up a bounded wait) are reported by
 * infini_attn_sync_status.  The result does not depend on the workspace's
 * previous contents, and repeated calls on the same inputs give bitwise
 * identical outputs. */
INFINI_API int infini_attn_forward(const void* q, const void* k, const void* v, const float* beta,
                        const float* M_in, const float* z_in, int seg_len, int rule,
                        const infini_dims_t* dims, void* out, float* M_out, float* z_out,
                        void* workspace, size_t workspace_bytes, void* stream);

/* The memory update alone: (M_out, z_out) = the state after the T segments
 * of k, v starting from (M_in, z_in), by `rule`, exactly as
 * infini_attn_forward computes them, without the attention output.
 * ("Hugging Face Infini-Attention 再現分析", Memory Update and State Transfer;
 * "Leave No Context Behind" explainer, "メモリの更新".)
 *   k, v             device, layouts above, element type dims->dtype
 *   M_in, z_in       device float32 state read by the first segment
 *   seg_len, rule    as for infini_attn_forward
 *   dims             as for infini_attn_forward; only B, H_kv, L, d_k, d_v
 *                    and dtype matter (H_q must still be a multiple of H_kv,
 *                    e.g. H_q = H_kv)
 *   M_out, z_out     device float32; may equal M_in / z_in (in place)
 *   workspace        as for infini_attn_forward, of
 *                    infini_attn_workspace_bytes(dims, seg_len, rule) bytes
 *   stream           cudaStream_t.
 * Under the linear rule the update is a sum over tokens, so the state of a
 * sequence cut at segment boundaries is M_0 plus the pieces' updates from a
 * zero state, added in order: the exchange step of a sequence-parallel
 * forward (one all-gather of every rank's update, then an exclusive prefix).
 * Errors: those of infini_attn_forward. */
INFINI_API int infini_attn_state_update(const void* k, const void* v, const float* M_in,
                                        const float* z_in, int seg_len, int rule,
                                        const infini_dims_t* dims, float* M_out, float* z_out,
                                        void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device workspace infini_attn_backward needs for these sizes (the
 * forward's per-segment states in fp32 and the per-query-head partials of
 * the backward).  0 if the arguments are invalid or the shape is not one the
 * backward supports. */
INFINI_API size_t infini_attn_backward_workspace_bytes(const infini_dims_t* dims, int seg_len,
                                                       int rule);

/* Backward of infini_attn_forward through the segments (back-propagation
 * through the memory, as training over a rollout of segments needs:
 * "Hugging Face Infini-Attention 再現分析", "重み減衰とロールアウト";
 * "Leave No Context Behind" explainer, "限界").  Given the gradients of a
 * scalar loss with respect to the forward's outputs, writes its gradients
 * with respect to the forward's inputs (the chain rule through every step of
 * the forward; rows whose retrieval denominator is exactly 0 carry none).
 *   q, k, v, beta,
 *   M_in, z_in,
 *   seg_len, rule,
 *   dims             the forward's arguments, unchanged
 *   dout             device [B, H_q, L, d_v], element type dims->dtype
 *   dM_out, dz_out   device float32 [B, H_kv, d_k, d_v] and [B, H_kv, d_k],
 *                    or NULL for a zero gradient
 *   dq               device float32 [B, H_q, L, d_k]
 *   dk, dv           device float32 [B, H_kv, L, d_k] / [B, H_kv, L, d_v]
 *   dbeta            device float32 [H_q]
 *   dM_in, dz_in     device float32, the shapes of M_in / z_in
 *   workspace        device scratch of infini_attn_backward_workspace_bytes
 *                    bytes, 256-byte aligned; or NULL with workspace_bytes == 0
 *                    (taken with cudaMallocAsync on `stream`, freed after)
 *   stream           cudaStream_t; asynchronous.
 * Supported: d_k == d_v in {32, 64} and seg_len <= 64 (the short-segment
 * training shapes); otherwise INFINI_ERR_UNSUPPORTED.  The outputs must not
 * overlap each other, the inputs or the workspace (INFINI_ERR_ALIAS); all
 * pointers 16-byte aligned (INFINI_ERR_ALIGN).  Every sum runs in a fixed
 * order: repeated calls give bitwise identical gradients.  Other errors:
 * INFINI_ERR_ARG, INFINI_ERR_WORKSPACE, INFINI_ERR_CUDA. */
INFINI_API int infini_attn_backward(const void* q, const void* k, const void* v, const float* beta,
                                    const float* M_in, const float* z_in, int seg_len, int rule,
                                    const infini_dims_t* dims, const void* dout,
                                    const float* dM_out, const float* dz_out, float* dq, float* dk,
                                    float* dv, float* dbeta, float* dM_in, float* dz_in,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* Sum of memory states: the exchange step of the sequence-parallel linear
 * rule, where the memory after a run of segments is the memory before it
 * plus the run's own update from a zero state ("Hugging Face
 * Infini-Attention 再現分析", Memory Update: the contributions accumulate).
 *   M_out = M_base + M(parts[0]) + ... + M(parts[n_parts - 1]),
 *   z_out = z_base + z(parts[0]) + ... + z(parts[n_parts - 1]),
 * every element added in fp32 in that order (bitwise deterministic).
 *   M_base, z_base   device float32 [B, H_kv, d_k, d_v] and [B, H_kv, d_k]
 *   parts            device float32, n_parts consecutive packed states, each
 *                    [M (B*H_kv*d_k*d_v floats) | z (B*H_kv*d_k floats)]
 *                    (the updates of infini_attn_state_update, gathered in
 *                    rank order); may be NULL when n_parts == 0
 *   n_parts          >= 0 (0 copies the base)
 *   M_out, z_out     device float32, shapes of M_base / z_base; may equal
 *                    M_base / z_base (in place); no other overlap
 *   stream           cudaStream_t; asynchronous.
 * All pointers must be memory of the current device and 16-byte aligned.
 * Errors: INFINI_ERR_ARG (NULL pointer, size < 1, n_parts < 0),
 * INFINI_ERR_ALIGN, INFINI_ERR_ALIAS, INFINI_ERR_CUDA. */
INFINI_API int infini_attn_state_sum(const float* M_base, const float* z_base, const float* parts,
                                     int n_parts, int B, int H_kv, int d_k, int d_v, float* M_out,
                                     float* z_out, void* stream);

/* Q/K/V projections with rotary position embedding: the prologue that
 * produces the heads the layer consumes.  The memory reuses the attention's
 * own Q, K and V ("Leave No Context Behind" explainer, "メモリ構造"); they
 * come from linear layers over the layer input ("Как работает
 * Infini-attention", section 9).  For every token row r = b L + t of x:
 *   y_r = x_r W^T + bias   (fp32 accumulation over d_model)
 * y's columns are H_q query heads, then H_kv key heads, then H_kv value heads
 * of d columns each.  Query and key heads are rotated (rotary embedding,
 * rotate-half pairing: for i < d/2, with c = rope_cos[t][i], s = rope_sin[t][i],
 *   y'_i = y_i c - y_{i+d/2} s,  y'_{i+d/2} = y_{i+d/2} c + y_i s);
 * value heads are not.  Results are rounded to bf16.
 *   x          device bf16 [B, L, d_model] (row-major, rows contiguous)
 *   w_qkv      device bf16 [(H_q + 2 H_kv) d, d_model]: W_q's rows, then
 *              W_k's, then W_v's (the layout of a linear layer's weight)
 *   bias       device float32 [(H_q + 2 H_kv) d], or NULL for none
 *   rope_cos, rope_sin
 *              device float32 [L, d/2] (row t rotates token t of every batch
 *              row; see infini_attn_rope_tables), or both NULL for no rotation
 *   dims       B, H_q, H_kv, L; d = d_k = d_v; dtype must be BF16
 *   d_model    input width
 *   q, k, v    device bf16 outputs [B, H_q, L, d], [B, H_kv, L, d],
 *              [B, H_kv, L, d]: the inputs of infini_attn_forward
 *   stream     cudaStream_t; asynchronous.
 * Supported: d_k == d_v in {64, 128}, d_model >= 64 and a multiple of 8,
 * dtype BF16 (otherwise INFINI_ERR_UNSUPPORTED).  The outputs must not
 * overlap each other or any input (INFINI_ERR_ALIAS); all pointers 16-byte
 * aligned (INFINI_ERR_ALIGN); one of rope_cos / rope_sin NULL without the
 * other, a NULL x / w_qkv / output, or a size < 1 is INFINI_ERR_ARG.  A kernel
 * that gives up a bounded wait sets the device status word (see
 * infini_attn_sync_status).  Other errors: INFINI_ERR_CUDA. */
INFINI_API int infini_attn_qkv_project(const void* x, const void* w_qkv, const float* bias,
                                       const float* rope_cos, const float* rope_sin,
                                       const infini_dims_t* dims, int d_model, void* q, void* k,
                                       void* v, void* stream);

/* Rotary embedding tables for infini_attn_qkv_project:
 *   cos_out[p][i] = cos(p base^(-2i/d)),  sin_out[p][i] = sin(p base^(-2i/d))
 * for p = 0..n_pos-1, i < d/2, computed in fp64 and rounded to float32
 * (RoFormer's frequencies; a reading, the pages name no position encoding).
 *   cos_out, sin_out   device float32 [n_pos, d/2], not overlapping
 *   n_pos >= 1, d >= 2 even, base > 0; stream: cudaStream_t.
 * Errors: INFINI_ERR_ARG (NULL, bad size or base), INFINI_ERR_ALIAS,
 * INFINI_ERR_CUDA. */
INFINI_API int infini_attn_rope_tables(float* cos_out, float* sin_out, int n_pos, int d,
                                       double base, void* stream);

/* Streaming decode: the layer forward one token at a time.  The current
 * segment's keys and values so far are kept by the caller in a rolling
 * buffer of seg_len rows per KV head; (M, z) hold the memory of the segments
 * before it.  Decoding a sequence token by token (pos = 0, 1, ..., S - 1,
 * 0, 1, ...) gives the outputs and states infini_attn_forward gives for the
 * whole sequence.  ("Hugging Face Infini-Attention 再現分析", State Transfer:
 * a stream processed segment by segment keeps only the memory; "Leave No
 * Context Behind" explainer, "実装上の流れ": read the memory, attend within the
 * segment, mix, update with the segment's K/V.)
 *
 * Bytes of device workspace infini_attn_decode_step needs (0 if the sizes are
 * invalid; dims->L is ignored).  The workspace starts with the step's ticket
 * counters: a workspace must be zero-filled before its first decode step
 * (each step leaves the counters at zero again); the rest is scratch. */
INFINI_API size_t infini_attn_decode_workspace_bytes(const infini_dims_t* dims, int seg_len,
                                                     int rule);

/* One decode step.
 *   q_t              device [B, H_q, d], element type dims->dtype: the new
 *                    token's queries
 *   k_t, v_t         device [B, H_kv, d]: its keys and values
 *   beta             device float32 [H_q]
 *   k_buf, v_buf     device [B, H_kv, seg_len, d]: rows 0..pos-1 hold the
 *                    current segment's earlier tokens; the call writes k_t,
 *                    v_t into row pos (rows after pos are not read)
 *   pos              0 <= pos < seg_len: the token's row in its segment
 *   M, z             device float32 [B, H_kv, d, d] and [B, H_kv, d]: the
 *                    state before the current segment.  When pos ==
 *                    seg_len - 1 the segment is complete and the call updates
 *                    them in place by `rule` with the whole buffer (after the
 *                    token's output); the next call starts a segment at pos 0.
 *                    At the end of a stream whose last segment is shorter,
 *                    infini_attn_state_update on the buffer's first pos + 1
 *                    rows (made contiguous) gives the final state.
 *   seg_len, rule    as for infini_attn_forward
 *   dims             B, H_q, H_kv, d_k = d_v = d, dtype; dims->L is ignored
 *   out_t            device [B, H_q, d], element type dims->dtype
 *   workspace        device scratch of infini_attn_decode_workspace_bytes
 *                    bytes, 256-byte aligned, zero-filled before its first
 *                    decode step (see above), or NULL with workspace_bytes
 *                    == 0 (stream-ordered allocation, zeroed by the call)
 *   stream           cudaStream_t.
 * The written regions (k_buf, v_buf, M, z, out_t) may not overlap each other,
 * the inputs or the workspace (INFINI_ERR_ALIAS); d_k != d_v is
 * INFINI_ERR_UNSUPPORTED.  Other errors: those of infini_attn_forward. */
INFINI_API int infini_attn_decode_step(const void* q_t, const void* k_t, const void* v_t,
                                       const float* beta, void* k_buf, void* v_buf, int pos,
                                       float* M, float* z, int seg_len, int rule,
                                       const infini_dims_t* dims, void* out_t, void* workspace,
                                       size_t workspace_bytes, void* stream);

/* Bytes of device arena infini_attn_forward_host needs: room for q, k, v,
 * beta, M, z, out and the workspace, each 256-byte aligned.  0 if invalid. */
INFINI_API size_t infini_attn_host_arena_bytes(const infini_dims_t* dims, int seg_len, int rule);

/* The same forward on HOST buffers.  q_h, k_h, v_h, beta_h, M_in_h, z_in_h,
 * out_h, M_out_h, z_out_h are host pointers with the layouts above (pinned
 * memory makes the copies asynchronous; pageable memory works but the copies
 * then synchronise).  `arena` is a device buffer of arena_bytes >=
 * infini_attn_host_arena_bytes(...), 256-byte aligned.  The call enqueues the
 * host-to-device copies, the forward and the device-to-host copies on
 * `stream`; the host results are valid once the stream has finished. */
INFINI_API int infini_attn_forward_host(const void* q_h, const void* k_h, const void* v_h,
                             const float* beta_h, const float* M_in_h, const float* z_in_h,
                             int seg_len, int rule, const infini_dims_t* dims,
                             void* out_h, float* M_out_h, float* z_out_h,
                             void* arena, size_t arena_bytes, void* stream);

/* Wait for `stream` to finish, then report and clear the device status word
 * the kernels set when one of their bounded waits ran out:
 * INFINI_OK, INFINI_ERR_TIMEOUT, INFINI_ERR_UNSUPPORTED if a kernel found
 * its dynamic shared memory placed where its layout cannot use it (it then
 * computes nothing), or INFINI_ERR_CUDA if the stream itself reported an
 * error. */
INFINI_API int infini_attn_sync_status(void* stream);

/* Benchmark support: per-kernel device timing.  While enabled, every
 * infini_attn_forward records a CUDA event on its stream before and after each
 * kernel it enqueues.  infini_attn_kernel_times waits for those events and
 * writes, for each kernel kind k < n_kinds, the summed milliseconds ms[k] and
 * the launch count launches[k] since the last reset (reset != 0 clears them).
 * Kinds: 0 = memory-state scan, 1 = segment attention.  The timing state is
 * process-wide; do not run forwards on other threads while reading it.
 * Errors: INFINI_ERR_ARG (NULL arrays, n_kinds < 1), INFINI_ERR_CUDA. */
INFINI_API int infini_attn_set_kernel_timing(int enable);
INFINI_API int infini_attn_kernel_times(double* ms, int* launches, int n_kinds, int reset);

/* No-allocation variant of infini_attn_forward.  The paper has no
 * counterpart: this is a deployment facility of this library.
 *
 * For callers that cannot allocate GPU memory while they run (code inside an
 * allocator callback, a loop that must never block on the driver's allocator,
 * an embedding that owns all device memory and cannot lend a workspace).
 * Arguments and results are those of infini_attn_forward without the
 * workspace: the scratch comes from one static device array of
 * infini_attn_noalloc_scratch_limit() bytes (64 MiB), which every GPU that
 * loads this part of the library holds until the process exits.
 *   - Problems whose workspace (infini_attn_workspace_bytes) exceeds that
 *     limit return INFINI_ERR_SCRATCH_LIMIT before anything is enqueued
 *     (a 1M-token stream does; the tiny, 200M-, 300M- and 8B-shaped
 *     workloads fit).
 *   - The call allocates nothing: no cudaMalloc, cudaMallocAsync or
 *     allocating library routine.  Every pointer must be memory of the
 *     current device, and the stream must belong to it.
 *   - Every call looks up the array's device address on the current device
 *     (cudaGetSymbolAddress); the address is not cached, so the call stays
 *     valid after cudaDeviceReset.
 *   - First call per device: CUDA loads GPU code lazily by default
 *     (CUDA_MODULE_LOADING=LAZY), so the first call on a device loads the
 *     library's modules it uses, which commits device memory for their code
 *     and for the 64 MiB array.  Make that first call as a warm-up, with the
 *     same shape, outside any region where allocation is forbidden and before
 *     any stream capture (or run the process with CUDA_MODULE_LOADING=EAGER).
 *     Later calls of that shape commit no device memory.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents; nothing in it needs clearing (every byte read is written
 *     earlier in the same call).  Calls whose GPU work overlaps -- on two
 *     streams, or from two threads -- race on the array and corrupt each
 *     other's results: serialise them.
 * Errors: those of infini_attn_forward, plus INFINI_ERR_SCRATCH_LIMIT. */
INFINI_API int infini_attn_forward_noalloc(const void* q, const void* k, const void* v,
                                           const float* beta, const float* M_in,
                                           const float* z_in, int seg_len, int rule,
                                           const infini_dims_t* dims, void* out, float* M_out,
                                           float* z_out, void* stream);

/* Bytes of the static scratch array infini_attn_forward_noalloc uses. */
INFINI_API size_t infini_attn_noalloc_scratch_limit(void);

/* Self-check of device approximations (a testing aid; the method has no
 * counterpart).  For i < n, with x, y_poly, y_mufu device float arrays and
 * bf16_bits a device uint32 array:
 *   y_poly[i]    = the FMA-pipe 2^x the attention kernel uses for part of its
 *                  probabilities (range reduction + degree-3 polynomial; inputs
 *                  below -125 are clamped to -125),
 *   y_mufu[i]    = the hardware 2^x approximation (subnormal results -> 0),
 *   bf16_bits[i] = bf16 bits of |x[i]| as the kernel packs probabilities
 *                  (round to nearest even).
 * Enqueued on `stream`.  Errors: INFINI_ERR_ARG, INFINI_ERR_CUDA. */
INFINI_API int infini_attn_selftest_approx(const float* x, float* y_poly, float* y_mufu,
                                           unsigned int* bf16_bits, int n, void* stream);

/* Self-check of the failure path of the tensor-core kernels' bounded waits (a
 * testing aid; the method has no counterpart).  Enqueues on `stream` one warp
 * that waits, through the same bounded mbarrier wait the kernels use, on a
 * barrier nothing ever arrives at: the wait gives up after its time limit
 * (2 s of %globaltimer), sets the timeout bit of the device status word and
 * the kernel returns normally -- no fault, the context stays usable.  A
 * following infini_attn_sync_status(stream) reports INFINI_ERR_TIMEOUT and
 * clears the word.  Errors: INFINI_ERR_CUDA (launch failed). */
INFINI_API int infini_attn_selftest_timeout(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* INFINI_ATTN_H */
