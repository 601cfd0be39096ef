/* A plain C99 caller of the layer's C ABI (host-side calls only, so it runs
 * without a GPU): the header compiles as C, the library links, and the
 * synchronous validation answers with the documented status codes. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "moe_lowbit.h"

static int failures = 0;

#define EXPECT(cond)                                              \
  do {                                                            \
    if (!(cond)) {                                                \
      fprintf(stderr, "line %d: %s\n", __LINE__, #cond);          \
      ++failures;                                                 \
    }                                                             \
  } while (0)

int main(void) {
  moe_dims_t decode = {1, 4096, 2048, 256, 8, 0, 0, 2048, 0};
  moe_dims_t prefill = {4096, 4096, 2048, 256, 8, 0, 0, 0, 0};
  moe_dims_t no_k = {4, 256, 128, 8, 0, 0, 0, 0, 0};
  size_t n_decode = moe_workspace_size(&decode);
  size_t n_prefill = moe_workspace_size(&prefill);
  static char ws_buf[512];
  char* ws = ws_buf + (256 - (uintptr_t)ws_buf % 256) % 256; /* 256-byte aligned, 256 bytes */
  moe_status_t st;

  EXPECT(n_decode > 0 && n_decode % 256 == 0);
  EXPECT(n_prefill > n_decode);
  EXPECT(moe_workspace_size(&no_k) == 0);

  st = moe_forward(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL);
  EXPECT(st == MOE_ERR_INVALID_ARG);
  EXPECT(strlen(moe_last_error_detail()) > 0);

  /* an expert slice past n_experts */
  st = moe_forward_partial(&decode, 0, decode.n_experts + 1, 1, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL,
                           NULL, NULL, NULL, NULL, ws, 256, NULL);
  EXPECT(st == MOE_ERR_INVALID_ARG);

  st = moe_permute(&no_k, NULL, NULL, NULL, NULL, ws, 256, NULL);
  EXPECT(st == MOE_ERR_INVALID_ARG);

  /* a workspace off the 256-byte alignment, then one too small */
  st = moe_route(&decode, NULL, NULL, NULL, NULL, NULL, NULL, NULL, ws + 16, 128, NULL);
  EXPECT(st == MOE_ERR_INVALID_ARG);
  st = moe_route(&decode, NULL, NULL, NULL, NULL, NULL, NULL, NULL, ws, 256, NULL);
  EXPECT(st == MOE_ERR_WORKSPACE);
  EXPECT(strcmp(moe_status_string(MOE_OK), moe_status_string(MOE_ERR_WORKSPACE)) != 0);

  EXPECT(moe_set_ffn_path(MOE_FFN_GEMV) == MOE_FFN_AUTO);
  EXPECT(moe_set_ffn_path(7) == -1);
  EXPECT(moe_set_ffn_path(MOE_FFN_AUTO) == MOE_FFN_GEMV);

  if (failures == 0) printf("ok %zu %zu\n", n_decode, n_prefill);
  return failures != 0;
}
