/* The C ABI used from plain C (no C++, no CUDA headers): every entry point
 * the header declares links, and argument errors come back as status codes
 * before anything touches a device.  Prints "ok" and exits 0 on success. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "flashnorm.h"

static int fails = 0;
#define EXPECT(cond)                                              \
  do {                                                            \
    if (!(cond)) {                                                \
      fprintf(stderr, "line %d: %s\n", __LINE__, #cond);          \
      ++fails;                                                    \
    }                                                             \
  } while (0)

int main(void) {
  /* fake, never dereferenced device addresses (16-byte aligned) */
  void* x = (void*)(uintptr_t)(1u << 20);
  void* w = (void*)(uintptr_t)(1u << 30);
  void* y = (void*)(uintptr_t)((uint64_t)1 << 34);
  void* ws = (void*)(uintptr_t)((uint64_t)1 << 36);
  float* part = (float*)(uintptr_t)((uint64_t)1 << 40);
  const float* gs = (const float*)(uintptr_t)((uint64_t)1 << 37);

  EXPECT(strncmp(fn_status_string(FN_ERR_ALIAS), "FN_", 3) == 0);
  EXPECT(fn_workspace_size(65, 4096, 6144, FN_W_BF16, 0) == 256);
  EXPECT(fn_workspace_size(1, 4096, 6144, FN_W_BF16, 0) > 256);

  EXPECT(fn_norm_proj(x, -1, 256, w, NULL, FN_W_BF16, 512, 1e-6f, y, ws, 1u << 30, NULL) == FN_ERR_INVALID_ARG);
  EXPECT(fn_norm_proj(x, 4, 100, w, NULL, FN_W_BF16, 512, 1e-6f, y, ws, 1u << 30, NULL) == FN_ERR_UNSUPPORTED_SHAPE);
  EXPECT(fn_norm_proj(x, 4, 256, w, NULL, FN_W_BF16, 512, 1e-6f, (char*)y + 2, ws, 1u << 30, NULL) ==
         FN_ERR_ALIGNMENT);
  EXPECT(fn_norm_proj(x, 4, 256, w, NULL, FN_W_BF16, 512, 1e-6f, (char*)x + 16, ws, 1u << 30, NULL) ==
         FN_ERR_ALIAS);
  EXPECT(fn_norm_proj(x, 0, 256, w, NULL, FN_W_BF16, 512, 1e-6f, NULL, NULL, 0, NULL) == FN_OK);
  EXPECT(fn_norm_proj_swiglu(x, 4, 256, w, NULL, FN_W_BF16, 512, -1.0f, y, ws, 1u << 30, NULL) ==
         FN_ERR_INVALID_ARG);
  EXPECT(fn_norm_proj_swiglu_nvfp4(x, 4, 256, w, NULL, FN_W_BF16, 512, 1e-6f, NULL, y, ws, ws, 1u << 30, NULL) ==
         FN_ERR_INVALID_ARG);
  EXPECT(fn_norm_proj_partial(x, 4, 256, w, NULL, FN_W_BF16, 512, NULL, ws, 1u << 30, NULL) == FN_ERR_INVALID_ARG);
  EXPECT(fn_post_scale(part, 4, 200, 0, 1024, 1e-6f, y, NULL) == FN_ERR_UNSUPPORTED_SHAPE);
  EXPECT(fn_fold_weights(x, NULL, NULL, 256, 512, FN_W_BF16, w, NULL, NULL) == FN_ERR_INVALID_ARG);
  EXPECT(fn_set_debug(99, 1) == FN_ERR_INVALID_ARG);
  EXPECT(fn_version() == 1);
  (void)gs;
  if (fails) return 1;
  printf("ok\n");
  return 0;
}
