/*
 * Uses the layer's C ABI from plain C (no Python, no torch types): the
 * workspace sizes of the V4-Flash layer, argument errors reported with a
 * message, and the encoder's argument checks.  None of these calls touches a
 * device, so the program runs without a GPU.  Exit status 0 when every check
 * holds; the failing check is printed otherwise.
 */
#include <stdio.h>
#include <string.h>

#include "moe.h"

static int failures = 0;

static void check(int ok, const char *what) {
  if (!ok) {
    printf("FAILED: %s (last error: %s)\n", what, moe_last_error());
    ++failures;
  }
}

int main(void) {
  moe_config c;
  memset(&c, 0, sizeof c);
  c.hidden = 4096;
  c.inter = 2048;
  c.n_experts = 256;
  c.top_k = 6;
  c.shared_inter = 2048;
  c.vocab = 129280;
  c.routed_scaling = 1.5f;
  c.rms_eps = 1e-6f;
  c.mode = MOE_ROUTE_ROUTER;
  c.flags = 0;
  c.routed_format = MOE_ROUTED_Q2;

  size_t persist = 0, s1 = 0, s32 = 0, s4096 = 0;
  check(moe_workspace_size(&c, 1, &persist, &s1) == MOE_OK, "workspace for one token");
  check(persist > 0 && s1 > 0, "non-zero sizes");
  check(moe_workspace_size(&c, MOE_SMALL_T_MAX, NULL, &s32) == MOE_OK && s32 >= s1, "workspace for 32 tokens");
  check(moe_workspace_size(&c, 4096, NULL, &s4096) == MOE_OK && s4096 >= s32, "workspace for 4096 tokens");

  c.routed_format = MOE_ROUTED_Q4K;
  size_t q4 = 0;
  check(moe_workspace_size(&c, 8, NULL, &q4) == MOE_OK && q4 > 0, "Q4_K workspace");
  c.routed_format = MOE_ROUTED_Q2;

  c.hidden = 4000;
  check(moe_workspace_size(&c, 1, NULL, NULL) == MOE_ERR_UNSUPPORTED_SHAPE, "hidden not a multiple of 256");
  check(strlen(moe_last_error()) > 0, "an error message");
  c.hidden = 4096;
  c.top_k = 9;
  check(moe_workspace_size(&c, 1, NULL, NULL) == MOE_ERR_UNSUPPORTED_SHAPE, "top_k above 8");
  c.top_k = 6;
  check(moe_workspace_size(&c, -1, NULL, NULL) == MOE_ERR_INVALID_ARG, "negative max_tokens");
  check(moe_workspace_size(NULL, 1, NULL, NULL) == MOE_ERR_INVALID_ARG, "NULL config");

  moe_handle *h = (moe_handle *)0x1;
  check(moe_init(&c, NULL, NULL, 0, NULL, &h) == MOE_ERR_INVALID_ARG && h == NULL, "init without weights");

  check(moe_quantize(7, NULL, 0, NULL, NULL, NULL) == MOE_ERR_INVALID_ARG, "unknown encoder format");
  check(moe_quantize(MOE_QUANT_Q2_K, NULL, 300, NULL, NULL, NULL) == MOE_ERR_UNSUPPORTED_SHAPE,
        "value count not a multiple of 256");
  check(moe_quantize(MOE_QUANT_Q8_0, NULL, 0, NULL, NULL, NULL) == MOE_OK, "no values: a no-op");

  check(moe_set_wait_limit(NULL, 100) == MOE_ERR_INVALID_ARG, "wait limit without a handle");

  /* expert parallelism: workspace sizes and argument checks */
  c.hidden = 4096;
  c.top_k = 6;
  c.n_experts = 256;
  size_t ed = 0, ex = 0, ec = 0;
  check(moe_ep_workspace_size(&c, 512, 3072, &ed, &ex, &ec) == MOE_OK && ed > 0 && ex > 0 && ec > 0,
        "expert-parallel workspace sizes");
  check(moe_ep_workspace_size(NULL, 1, 1, NULL, NULL, NULL) == MOE_ERR_INVALID_ARG, "EP workspace without config");
  check(moe_ep_workspace_size(&c, -1, 1, NULL, NULL, NULL) == MOE_ERR_INVALID_ARG, "EP negative tokens");
  c.flags = MOE_FLAG_EXPERTS_ONLY | MOE_FLAG_NO_ROUTED;
  check(moe_workspace_size(&c, 1, NULL, NULL) == MOE_ERR_INVALID_ARG, "exclusive EP flags");
  c.flags = 0;
  check(moe_ep_dispatch(NULL, NULL, NULL, 1, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) == MOE_ERR_INVALID_ARG,
        "dispatch without a handle");
  check(moe_ep_experts(NULL, NULL, NULL, NULL, 1, 0, NULL, NULL, 0, NULL) == MOE_ERR_INVALID_ARG,
        "experts without a handle");
  check(moe_ep_combine(NULL, NULL, 1, NULL, NULL, NULL, NULL, 0, NULL) == MOE_ERR_INVALID_ARG,
        "combine without a handle");

  moe_destroy(NULL);
  if (failures == 0) printf("C ABI checks passed\n");
  return failures == 0 ? 0 : 1;
}
