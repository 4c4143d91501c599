/* A plain C11 caller of the library: the header compiles as C, the symbols
 * link, and the host-side entry points behave as documented without a GPU
 * (argument validation happens before any device call).  Prints "ok" and
 * returns 0 on success; prints the failing check and returns 1 otherwise. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "lora_gemm.h"

#define CHECK(cond)                                   \
  do {                                                \
    if (!(cond)) {                                    \
      printf("failed: %s (line %d)\n", #cond, __LINE__); \
      return 1;                                       \
    }                                                 \
  } while (0)

int main(void) {
  void* const x = (void*)(uintptr_t)0x7F0000000000ull; /* fake, aligned, never dereferenced */
  void* const w = (void*)(uintptr_t)0x7F0001000000ull;
  float* const z = (float*)(uintptr_t)0x7F0002000000ull;
  void* const mis = (void*)(uintptr_t)0x7F0000000004ull;

  CHECK(lg_version() >= 10000);
  CHECK(strcmp(lg_status_string(LG_OK), lg_status_string(LG_ERR_CUDA)) != 0);
  CHECK(lg_lora_linear_workspace_size(10, 7168, 7168, 576) == 2u * (2u * 576u * 7168u));
  CHECK(lg_lora_linear_workspace_size(10, 100, 64, 64) == 0);
  CHECK(lg_mx_scale_bytes(1, 128) == 512);
  CHECK(lg_lora_linear(x, w, NULL, NULL, NULL, 256, 128, 128, 0, NULL, 0, NULL) == LG_ERR_INVALID_ARG);
  CHECK(lg_lora_linear(x, w, NULL, NULL, x, 0, 128, 128, 0, NULL, 0, NULL) == LG_OK);
  CHECK(lg_lora_linear(mis, w, NULL, NULL, z, 256, 128, 128, 0, NULL, 0, NULL) == LG_ERR_MISALIGNED);
  CHECK(lg_euler_step(z, z, 16, 0.909f, 0.857f, NULL) == LG_ERR_INVALID_ARG); /* x and v overlap */
  CHECK(lg_lora_linear_euler(x, w, NULL, NULL, z, NULL, 256, 128, 24, 0, 100, 0.857f, 0.667f, NULL, 0, NULL) ==
        LG_ERR_INVALID_ARG); /* M not a multiple of the frame */
  CHECK(lg_set_cluster_size(3) == LG_ERR_INVALID_ARG);
  CHECK(lg_set_cluster_size(0) == LG_OK);

  {
    float sig[16];
    int n = 0;
    CHECK(lg_shift_ladder(0.923f, 8, 12.0, sig, 16, &n) == LG_OK);
    CHECK(n == 5 && sig[0] == 0.923f && sig[n - 1] == 0.0f);
  }
  printf("ok\n");
  return 0;
}
