/* A plain C99 consumer of include/convrot.h: compiles against the header
 * alone, links libconvrot.so, and exercises calls that need no GPU (argument
 * checks return before any launch).  Exit status 0 when every check holds. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "convrot.h"

#define EXPECT(cond)                                             \
  do {                                                           \
    if (!(cond)) {                                               \
      fprintf(stderr, "%s:%d: %s\n", __FILE__, __LINE__, #cond); \
      return 1;                                                  \
    }                                                            \
  } while (0)

int main(void) {
  uint8_t buf[64 + 16];
  void* fake = (void*)(((uintptr_t)buf + 15) & ~(uintptr_t)15); /* 16-byte aligned, never dereferenced */

  EXPECT(convrot_version() > 0);
  EXPECT(convrot_workspace_bytes(CONVROT_OP_LINEAR_INT8, 4608, 11520, 3840) >= 4608u * 3840u);
  EXPECT(convrot_workspace_bytes(CONVROT_OP_LINEAR_INT8_SLICED, 4608, 1024, 3840) <
         convrot_workspace_bytes(CONVROT_OP_LINEAR_INT8, 4608, 1024, 3840));
  EXPECT(convrot_workspace_bytes(99, 1, 1, 1) == 0);
  EXPECT(convrot_noalloc_scratch_bytes() == CONVROT_NOALLOC_SCRATCH_BYTES);

  /* a rotation needs a G in {4, 16, 64, 256} */
  convrot_rotation_t R = NULL;
  float r3[9] = {1, 0, 0, 0, 1, 0, 0, 0, 1};
  EXPECT(convrot_rotation_create(r3, 3, &R) == CONVROT_ERR_UNSUPPORTED);
  EXPECT(R == NULL);
  EXPECT(strlen(convrot_last_error_string()) > 0);

  /* argument errors return before any launch */
  EXPECT(convrot_rotate_quant_act(NULL, 4, 256, NULL, NULL, NULL, NULL) == CONVROT_ERR_INVALID_ARG);
  EXPECT(convrot_int8_gemm_s32((const int8_t*)fake, (const int8_t*)fake, 8, 20, 64,
                               (int32_t*)fake, NULL) == CONVROT_ERR_INVALID_ARG); /* N % 16 != 0 */
  EXPECT(convrot_int8_gemm_f16((const int8_t*)fake, (const float*)fake, (const int8_t*)fake,
                               (const float*)fake, 1, NULL, 0, 32, 64, (convrot_f16*)fake,
                               NULL) == CONVROT_OK); /* M = 0: nothing to do */
  EXPECT(convrot_selftest_wait_timeout(0, NULL) == CONVROT_ERR_INVALID_ARG);

  /* the default path and the checked forward */
  EXPECT(convrot_workspace_bytes(CONVROT_OP_LINEAR_DEQUANT, 64, 1024, 512) == 2u * 1024u * 512u);
  EXPECT(convrot_workspace_bytes(CONVROT_OP_LINEAR_CHECKED, 4608, 1024, 512) >=
         convrot_workspace_bytes(CONVROT_OP_LINEAR_DEQUANT, 4608, 1024, 512) +
             2u * CONVROT_CHECK_ROWS * 1024u);
  EXPECT(convrot_dense_linear((const convrot_bf16*)fake, 8, 64, 24, (const convrot_bf16*)fake, NULL,
                              (convrot_bf16*)fake, NULL) == CONVROT_ERR_INVALID_ARG);
  int path = -1, latched = -1, keys = -1;
  EXPECT(convrot_linear_checked((const convrot_bf16*)fake, 8, 256, 32, NULL, (const int8_t*)fake,
                                (const float*)fake, 1, NULL, (convrot_bf16*)fake, fake, 1u << 24,
                                &path, NULL) == CONVROT_ERR_INVALID_ARG);
  EXPECT(path == 0);
  EXPECT(convrot_check_state(0, &latched, &keys) == CONVROT_OK && latched == 0 && keys == 0);
  EXPECT(convrot_check_set_min_cosine(2.0) == CONVROT_ERR_INVALID_ARG);
  EXPECT(convrot_check_min_cosine() == 0.99);
  EXPECT(CONVROT_PATH_INT8 != CONVROT_PATH_DEQUANT);
  convrot_check_reset();
  printf("c abi ok\n");
  return 0;
}
