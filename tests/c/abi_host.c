/* Plain-C client of libmoe_b200.so: the header compiles as C99 and the
 * host-side entry points (no GPU work) behave as documented.  Exit code 0
 * on success; the first failed check prints its line and exits 1. */
#include <stdio.h>
#include <string.h>

#include "moe.h"

#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      fprintf(stderr, "abi_host.c:%d: check failed: %s\n", __LINE__, #cond); \
      return 1;                                                       \
    }                                                                 \
  } while (0)

int main(void) {
  CHECK(strstr(moe_version(), "sm_100a") != NULL);
  CHECK(strcmp(moe_status_string(MOE_OK), "MOE_OK") == 0);
  CHECK(strncmp(moe_status_string(MOE_ERR_DEVICE_TIMEOUT), "MOE_ERR_DEVICE_TIMEOUT", 22) == 0);

  /* capacity: ceil(T * k * cf / E) in exact integers */
  CHECK(moe_expert_capacity(8192, 2, 64, 6, 5) == 308);
  CHECK(moe_expert_capacity(64, 2, 8, 0, 1) == 0);
  CHECK(moe_expert_capacity(64, 2, 8, 1, 0) == -1);

  MoEConfig c;
  memset(&c, 0, sizeof c);
  c.num_experts = 8;
  c.top_k = 2;
  c.hidden_dim = 128;
  c.intermediate_dim = 256;
  c.gate = MOE_GATE_SOFTMAX_TOPK_RENORM;
  c.clamp_mode = MOE_CLAMP_PREACT;
  c.act_dtype = MOE_BF16;
  c.expert_dtype = MOE_BF16;
  c.out_dtype = MOE_F32;
  CHECK(moe_workspace_size(&c, 64) > 0);
  CHECK(moe_workspace_size(&c, 4096) > moe_workspace_size(&c, 64));
  CHECK(moe_dispatch_workspace_size(&c, 64) >= 256);

  /* argument errors come back synchronously, before any CUDA work */
  MoEWeights w;
  memset(&w, 0, sizeof w);
  int32_t idx[4];
  float tw[4];
  unsigned char ws[256];
  CHECK(moe_route_topk(NULL, 4, (void *)16, &w, NULL, idx, tw, ws, sizeof ws, NULL) == MOE_ERR_INVALID_ARG);
  c.top_k = 9;
  CHECK(moe_workspace_size(&c, 64) == 0);
  CHECK(moe_route_topk(&c, 4, (void *)16, &w, NULL, idx, tw, ws, sizeof ws, NULL) == MOE_ERR_INVALID_ARG);
  c.top_k = 2;
  CHECK(moe_forward_profiled(&c, 64, (void *)16, &w, NULL, (void *)16, NULL, NULL, ws, sizeof ws, NULL, NULL, 3) ==
        MOE_ERR_INVALID_ARG);
  CHECK(moe_selftest_wait_timeout(NULL, 256, NULL) == MOE_ERR_INVALID_ARG);
  CHECK(moe_check_device_status(NULL, NULL) == MOE_ERR_INVALID_ARG);
  printf("abi_host: ok\n");
  return 0;
}
