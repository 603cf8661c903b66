/* A plain C caller of the decoder's C ABI (no Python, no torch): the
 * argument checks that need no GPU.  Built and run by tests/test_abi_c_cpu.py;
 * exits 0 when every check holds, else prints the failed check and exits 1. */
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "fdllm.h"

#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      return 1;                                                       \
    }                                                                 \
  } while (0)

static fdllm_config tiny(void) {
  fdllm_config c;
  memset(&c, 0, sizeof c);
  c.n_layers = 2;
  c.d_model = 128;
  c.n_heads = 4;
  c.n_kv_heads = 4;
  c.head_dim = 32;
  c.ffn_dim = 384;
  c.vocab = 512;
  c.mask_id = 511;
  c.rope_theta = 1e4f;
  c.rms_eps = 1e-5f;
  c.logit_scale = 8.0f;
  c.dtype = FDLLM_DTYPE_F32;
  c.max_batch = 1;
  c.max_seq = 96;
  return c;
}

int main(void) {
  fdllm_ctx* ctx = NULL;
  /* NULL config and NULL out */
  CHECK(fdllm_create(NULL, 0, NULL, NULL, &ctx) == FDLLM_ERR_ARG);
  CHECK(ctx == NULL);
  CHECK(fdllm_last_error(NULL) != NULL && strlen(fdllm_last_error(NULL)) > 0);
  /* configs the header rules out are rejected before any device work */
  fdllm_config c = tiny();
  c.d_model = 100;
  CHECK(fdllm_create(&c, 0, NULL, NULL, &ctx) == FDLLM_ERR_ARG && ctx == NULL);
  c = tiny();
  c.mask_id = c.vocab;
  CHECK(fdllm_create(&c, 0, NULL, NULL, &ctx) == FDLLM_ERR_ARG && ctx == NULL);
  c = tiny();
  c.logit_scale = NAN;
  CHECK(fdllm_create(&c, 0, NULL, NULL, &ctx) == FDLLM_ERR_ARG && ctx == NULL);
  c = tiny();
  c.max_batch = 65;
  CHECK(fdllm_create(&c, 0, NULL, NULL, &ctx) == FDLLM_ERR_ARG && ctx == NULL);
  /* an allocator with only one of its two functions */
  fdllm_allocator half;
  memset(&half, 0, sizeof half);
  c = tiny();
  CHECK(fdllm_create(&c, 0, NULL, &half, &ctx) == FDLLM_ERR_ARG && ctx == NULL);
  /* calls on a NULL context */
  int steps = -1;
  int32_t out[16];
  CHECK(fdllm_load_weights(NULL, NULL, 0) == FDLLM_ERR_ARG);
  CHECK(fdllm_generate(NULL, NULL, 0, 16, 16, 0.9f, FDLLM_CACHE_DUAL, out, &steps, NULL) ==
        FDLLM_ERR_ARG);
  CHECK(fdllm_inexact_weight_count(NULL) == -1);
  CHECK(fdllm_destroy(NULL) == FDLLM_OK);
  printf("abi_smoke ok\n");
  return 0;
}
