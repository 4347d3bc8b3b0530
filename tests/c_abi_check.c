/* A plain C99 consumer of include/infini_attn.h and libinfini_attn.so: the
 * boundary has to be usable without C++ or PyTorch.  Runs without a GPU: it
 * only makes calls that are answered on the host (version, status strings,
 * sizing, planning, argument checks), and prints "c-abi ok" when every answer
 * is the documented one.  Compiled and run by tests/test_abi_cpu.py. */
#include <stdio.h>
#include <string.h>

#include "infini_attn.h"

static int failures = 0;

static void expect(int cond, const char* what) {
  if (!cond) {
    fprintf(stderr, "FAILED: %s\n", what);
    ++failures;
  }
}

int main(void) {
  expect((infini_attn_version() >> 16) == 1, "major version 1");
  for (int s = -8; s <= 0; ++s) {
    const char* msg = infini_attn_status_string(s);
    expect(msg != NULL && strlen(msg) > 0, "status string");
  }

  /* The 8B-shaped workload: bf16, GQA 32/8, d = 128, 2048-token segments. */
  infini_dims_t d8b = {2, 32, 8, 32768, 128, 128, INFINI_DTYPE_BF16};
  infini_plan_t plan;
  expect(infini_attn_plan(&d8b, 2048, INFINI_RULE_DELTA, &plan) == INFINI_OK, "plan 8B");
  expect(plan.path == INFINI_PATH_TCGEN05, "8B runs on the tensor cores");
  expect(plan.num_segments == 16, "16 segments");
  expect(plan.workspace_bytes == infini_attn_workspace_bytes(&d8b, 2048, INFINI_RULE_DELTA),
         "plan and sizing agree");
  expect(plan.workspace_bytes >= (size_t)16 * 2 * 8 * 128 * 4, "workspace holds z per segment");

  /* fp32 I/O runs on the CUDA cores. */
  infini_dims_t dsm = {1, 2, 2, 256, 32, 32, INFINI_DTYPE_F32};
  expect(infini_attn_plan(&dsm, 64, INFINI_RULE_LINEAR, &plan) == INFINI_OK, "plan tiny");
  expect(plan.path == INFINI_PATH_SIMT, "fp32 runs on the CUDA cores");

  /* Invalid sizes: reported, nothing enqueued. */
  infini_dims_t bad = d8b;
  bad.H_q = 30; /* not a multiple of H_kv */
  expect(infini_attn_plan(&bad, 2048, INFINI_RULE_DELTA, &plan) == INFINI_ERR_ARG, "H_q % H_kv");
  expect(infini_attn_workspace_bytes(&bad, 2048, INFINI_RULE_DELTA) == 0, "no workspace for bad sizes");
  bad = d8b;
  bad.d_k = 96;
  expect(infini_attn_plan(&bad, 2048, INFINI_RULE_DELTA, &plan) == INFINI_ERR_UNSUPPORTED, "d_k 96");
  expect(infini_attn_plan(&d8b, 0, INFINI_RULE_DELTA, &plan) == INFINI_ERR_ARG, "seg_len 0");
  expect(infini_attn_plan(&d8b, 2048, 7, &plan) == INFINI_ERR_ARG, "unknown rule");

  /* Entry points reject NULL pointers before touching a GPU. */
  expect(infini_attn_forward(NULL, NULL, NULL, NULL, NULL, NULL, 2048, INFINI_RULE_DELTA, &d8b, NULL,
                             NULL, NULL, NULL, 0, NULL) == INFINI_ERR_ARG,
         "forward NULL");
  expect(infini_attn_qkv_project(NULL, NULL, NULL, NULL, NULL, &d8b, 4096, NULL, NULL, NULL, NULL) ==
             INFINI_ERR_ARG,
         "projection NULL");
  expect(infini_attn_rope_tables(NULL, NULL, 16, 128, 10000.0, NULL) == INFINI_ERR_ARG, "tables NULL");
  expect(infini_attn_backward_workspace_bytes(&d8b, 2048, INFINI_RULE_DELTA) == 0,
         "no backward for 2048-token segments");

  if (failures) return 1;
  printf("c-abi ok\n");
  return 0;
}
