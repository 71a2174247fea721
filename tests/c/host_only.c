/* A plain C caller of the library: the header compiles as C99 and the entry points that
 * need no GPU behave as include/moe.h says (workspace sizing, argument checks before any
 * launch, status strings).  Exits 0 when every check holds, else prints the first failure. */
#include <stdio.h>
#include <string.h>

#include "moe.h"

#define CHECK(cond)                                                        \
  do {                                                                     \
    if (!(cond)) {                                                         \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond);  \
      return 1;                                                            \
    }                                                                      \
  } while (0)

int main(void) {
  moe_config cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.max_tokens = 256;
  cfg.hidden = 7168;
  cfg.num_experts = 48;
  cfg.top_k_max = 3;
  cfg.inter = 5120;
  cfg.num_shared = 1;
  cfg.shared_inter = 5120;
  cfg.renormalize = 1;
  cfg.wtype = MOE_W_BF16;

  moe_plan_t plan = NULL;
  size_t ws = 0;
  CHECK(moe_plan_create(&cfg, &plan, &ws) == MOE_OK);
  CHECK(plan != NULL && ws > 0 && ws % 256 == 0);

  /* a larger batch needs a larger workspace */
  moe_config big = cfg;
  big.max_tokens = 512;
  moe_plan_t plan2 = NULL;
  size_t ws2 = 0;
  CHECK(moe_plan_create(&big, &plan2, &ws2) == MOE_OK && ws2 > ws);
  moe_plan_destroy(plan2);

  /* shapes the library does not take are refused on the host */
  moe_config bad = cfg;
  bad.inter = 100;
  moe_plan_t p3 = NULL;
  CHECK(moe_plan_create(&bad, &p3, &ws2) == MOE_ERR_UNSUPPORTED && p3 == NULL);
  bad = cfg;
  bad.top_k_max = 9;
  CHECK(moe_plan_create(&bad, &p3, &ws2) != MOE_OK);
  CHECK(moe_plan_create(NULL, &p3, &ws2) == MOE_ERR_INVALID_ARG);

  /* argument errors come back before anything is enqueued (there is no GPU here) */
  moe_weights w;
  memset(&w, 0, sizeof w);
  w.router_w = (const float *)0x1000;
  w.w_gate_up = (const void *)0x2000;
  w.w_down = (const void *)0x3000;
  w.ws_gate_up = (const void *)0x4000;
  w.ws_down = (const void *)0x5000;
  void *x = (void *)0x6000, *out = (void *)0x7000, *wsp = (void *)0x100000;
  CHECK(moe_forward(plan, &w, x, NULL, 257, 3, out, wsp, ws, NULL, NULL) == MOE_ERR_INVALID_ARG);
  CHECK(moe_forward(plan, &w, x, NULL, 16, 4, out, wsp, ws, NULL, NULL) == MOE_ERR_INVALID_ARG);
  CHECK(moe_forward(plan, &w, x, NULL, 16, 3, out, wsp, ws - 1, NULL, NULL) == MOE_ERR_WORKSPACE);
  CHECK(moe_forward(plan, &w, x, NULL, 16, 3, (void *)0x7008, wsp, ws, NULL, NULL) ==
        MOE_ERR_INVALID_ARG);
  CHECK(moe_forward(plan, &w, x, NULL, 0, 3, out, wsp, ws, NULL, NULL) == MOE_OK);
  float *dst[2] = {(float *)0x8000, (float *)0x9000};
  CHECK(moe_forward_scatter(plan, &w, x, NULL, 16, 3, dst, 2, 7, 0, wsp, ws, NULL, NULL) ==
        MOE_ERR_INVALID_ARG);                                   /* 2 * 7 != 16 */
  CHECK(moe_forward_scatter_experts(plan, &w, x, NULL, 16, 3, dst, 2, 8, 0, 40, 49, wsp, ws,
                                    NULL, NULL) == MOE_ERR_INVALID_ARG);   /* range past E */
  CHECK(moe_reduce_partials((const float *)0x8000, 0, 4, 7168, NULL, out, NULL) ==
        MOE_ERR_INVALID_ARG);
  CHECK(moe_forward(NULL, &w, x, NULL, 16, 3, out, wsp, ws, NULL, NULL) == MOE_ERR_INVALID_ARG);

  /* the host-buffer pipeline: slot sizes, and refusals before any CUDA call */
  size_t slot_bytes = 0;
  CHECK(moe_pipeline_slot_bytes(plan, 16, 3, &slot_bytes) == MOE_OK && slot_bytes > 0);
  CHECK(moe_pipeline_slot_bytes(plan, 0, 3, &slot_bytes) == MOE_ERR_INVALID_ARG);
  moe_pipeline_t pipe = (moe_pipeline_t)0x1;
  CHECK(moe_pipeline_create(plan, &w, 3, 16, 3, 1, (void *)0x200000, slot_bytes - 1, wsp, ws,
                            &pipe) == MOE_ERR_WORKSPACE && pipe == NULL);
  CHECK(moe_pipeline_create(plan, &w, 4, 16, 3, 1, (void *)0x200000, slot_bytes, wsp, ws,
                            &pipe) == MOE_ERR_INVALID_ARG && pipe == NULL);
  CHECK(moe_pipeline_submit(NULL, x, NULL, out) == MOE_ERR_INVALID_ARG);
  moe_pipeline_destroy(NULL);

  CHECK(moe_plan_set_wait_limit(NULL, 1) == MOE_ERR_INVALID_ARG);
  CHECK(moe_plan_set_wait_limit(plan, 5000000000ull) == MOE_OK);

  CHECK(strlen(moe_status_string(MOE_OK)) > 0);
  CHECK(strcmp(moe_status_string(MOE_ERR_WORKSPACE), moe_status_string(MOE_OK)) != 0);
  CHECK(moe_last_cuda_error_string() != NULL);

  moe_plan_destroy(plan);
  puts("host-only C checks passed");
  return 0;
}
