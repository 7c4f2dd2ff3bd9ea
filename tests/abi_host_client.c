/* A plain C client of the library: it includes include/moe.h as C99, links
   libmoe_b200.so and exercises the entry points that need no GPU (sizes,
   capacities, status strings, host-side argument checks).  Built and run by
   tests/test_abi_c.py; prints "ok" on success. */
#include <stdio.h>
#include <string.h>

#include "moe.h"

static int fails = 0;
#define CHECK(cond)                                             \
  do {                                                          \
    if (!(cond)) {                                              \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      ++fails;                                                  \
    }                                                           \
  } while (0)

int main(void) {
  moe_config c;
  memset(&c, 0, sizeof c);
  c.T = 2048;
  c.d_model = 4096;
  c.n_experts = 8;
  c.top_k = 2;
  c.d_ff = 14336;
  c.dtype = MOE_BF16;
  c.gating = MOE_SOFTMAX_TOPK;
  c.expert_act = MOE_ACT_SWIGLU;
  c.weight_format = MOE_W_NATIVE;

  const size_t ws = moe_workspace_bytes(&c);
  CHECK(ws > (size_t)c.T * c.top_k * c.d_model * 2); /* holds at least the dispatched rows */
  CHECK(moe_expert_capacity(&c) == c.T * c.top_k);   /* dropless */
  c.capacity_factor = 1.0f;
  CHECK(moe_expert_capacity(&c) == 512);             /* ceil(2048 * 2 / 8 * 1.0) */
  c.capacity_factor = 0.0f;

  CHECK(strcmp(moe_status_string(MOE_OK), "ok") == 0);
  CHECK(moe_status_string(MOE_ERR_TIMEOUT) != NULL);
  CHECK(moe_e4m3_weight_bytes(3, 16) == 256 + 3 * sizeof(float)); /* codes padded to 256 B, then scales */
  CHECK(moe_e4m3_weight_bytes(3, 15) == 0);                        /* rows must be whole 16-byte lines */

  /* host checks reject before launching anything */
  moe_config bad = c;
  bad.top_k = 9; /* k > E */
  CHECK(moe_workspace_bytes(&bad) == 0);
  CHECK(moe_forward(&c, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) ==
        MOE_ERR_INVALID_ARG);

  if (fails) return 1;
  printf("ok\n");
  return 0;
}
