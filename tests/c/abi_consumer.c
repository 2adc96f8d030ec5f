/*
 * A plain C99 consumer of the library's C ABI (include/fa.h), built and run by
 * tests/test_c_consumer.py on a machine without a GPU. It shows that the header is valid C
 * with no C++ or framework types, that a C program links against libfa_b200.so, and that
 * the host-side contract holds without Python: status strings, workspace sizes, and
 * argument errors returned before any CUDA call. No tensor is ever dereferenced: every
 * call that takes tensors carries one fault.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "fa.h"

static int failures = 0;

#define EXPECT(cond)                                                   \
  do {                                                                 \
    if (!(cond)) {                                                     \
      fprintf(stderr, "FAILED line %d: %s\n", __LINE__, #cond);        \
      ++failures;                                                      \
    }                                                                  \
  } while (0)

/* Stand-in device addresses: 16-byte aligned, never dereferenced. */
#define PTR(x) ((void*)(uintptr_t)(x))

int main(void) {
  void* q = PTR(0x1000);
  void* k = PTR(0x2000);
  void* v = PTR(0x3000);
  void* o = PTR(0x4000);
  float* lse = (float*)PTR(0x5000);
  int* lens = (int*)PTR(0x6000);
  size_t ws_need;

  EXPECT(strcmp(fa_status_string(FA_OK), "FA_OK") == 0);
  EXPECT(strcmp(fa_status_string(FA_ERR_WORKSPACE), "FA_ERR_WORKSPACE") == 0);
  EXPECT(strstr(fa_build_info(), "sm_100a") != NULL);

  /* fa_fwd: one fault per call. */
  EXPECT(fa_fwd(NULL, k, v, o, lse, 1, 2, 1, 64, 64, 64, 1, 0.125f, FA_FP16, NULL) ==
         FA_ERR_INVALID_ARG);
  EXPECT(fa_fwd(q, k, v, o, lse, 1, 3, 2, 64, 64, 64, 1, 0.125f, FA_FP16, NULL) ==
         FA_ERR_INVALID_ARG);
  EXPECT(fa_fwd(q, k, v, o, lse, 1, 2, 1, 64, 64, 64, 1, -1.0f, FA_FP16, NULL) ==
         FA_ERR_INVALID_ARG);
  EXPECT(fa_fwd(q, k, v, o, lse, 1, 2, 1, 64, 64, 96, 1, 0.125f, FA_FP16, NULL) ==
         FA_ERR_UNSUPPORTED);
  EXPECT(fa_fwd(q, k, v, o, lse, 1, 2, 1, 64, 64, 64, 1, 0.125f, (fa_dtype)7, NULL) ==
         FA_ERR_UNSUPPORTED);
  EXPECT(fa_fwd(q, PTR(0x2008), v, o, lse, 1, 2, 1, 64, 64, 64, 1, 0.125f, FA_BF16, NULL) ==
         FA_ERR_ALIGNMENT);

  /* Workspace sizes are pure host arithmetic. */
  ws_need = fa_decode_workspace_bytes(64, 32, 4096, 128);
  EXPECT(ws_need >= (size_t)64 * 32 * (128 + 1) * 4 && ws_need % 256 == 0);
  EXPECT(fa_decode_workspace_bytes(0, 32, 4096, 128) == 0);
  EXPECT(fa_bwd_workspace_bytes(1, 2, 200) == (size_t)2 * 2 * 256 * 4);
  EXPECT(fa_bwd_workspace_bytes(1, 2, 0) == 0);

  /* fa_decode: a missing or short workspace, a misaligned length vector. */
  EXPECT(fa_decode(q, k, v, lens, o, NULL, 64, 32, 8, 4096, 128, 0.088f, FA_BF16, NULL, 0,
                   NULL) == FA_ERR_WORKSPACE);
  EXPECT(fa_decode(q, k, v, lens, o, NULL, 64, 32, 8, 4096, 128, 0.088f, FA_BF16, PTR(0x7000),
                   ws_need - 1, NULL) == FA_ERR_WORKSPACE);
  EXPECT(fa_decode(q, k, v, (int*)PTR(0x6002), o, NULL, 64, 32, 8, 4096, 128, 0.088f, FA_BF16,
                   PTR(0x7000), ws_need, NULL) == FA_ERR_ALIGNMENT);

  /* fa_bwd requires the LSE; fa_fwd_fp8 requires positive descales and d = 128. */
  EXPECT(fa_bwd(q, k, v, o, NULL, q, q, k, v, 1, 2, 1, 200, 200, 64, 1, 0.125f, FA_FP16,
                PTR(0x7000), fa_bwd_workspace_bytes(1, 2, 200), NULL) == FA_ERR_INVALID_ARG);
  EXPECT(fa_fwd_fp8(q, k, v, o, lse, 1, 2, 1, 128, 128, 128, 1, 0.088f, 0.0f, 1.0f, 1.0f,
                    NULL) == FA_ERR_INVALID_ARG);
  EXPECT(fa_fwd_fp8(q, k, v, o, lse, 1, 2, 1, 128, 128, 64, 1, 0.088f, 1.0f, 1.0f, 1.0f,
                    NULL) == FA_ERR_UNSUPPORTED);

  /* Paged pool: a page size that is not a power of two. */
  EXPECT(fa_decode_paged(q, k, v, lens, lens, o, NULL, 2, 8, 2, 40, 48, 16, 128, 0.088f,
                         FA_BF16, PTR(0x7000), ws_need, NULL) == FA_ERR_UNSUPPORTED);

  if (failures) {
    fprintf(stderr, "%d check(s) failed\n", failures);
    return 1;
  }
  printf("C ABI consumer: all checks passed\n");
  return 0;
}
