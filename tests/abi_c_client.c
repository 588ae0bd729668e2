/* A plain C99 client of libcsa.so: it compiles against include/csa.h alone,
 * links the library and exercises host-side validation and the workspace
 * queries.  Every call below fails validation before anything is launched,
 * so it runs without a GPU. */
#include <stdio.h>

#include "csa.h"

int main(void) {
  csa_params p = {2, 512, 64, 4, 64, 128, 512, 64, 128, CSA_KV_FP8_BF16, CSA_IDX_MXFP4, CSA_ACT_BF16,
                  0.044f, 10000.0f, 1e-6f};
  csa_params bad = p;
  void* A = (void*)0x10000; /* fake, 16-byte aligned: validation fails first */
  csa_kv kv = {A, (float*)A, 100};
  bad.d = 256;
  csa_status s_null = csa_index_topk(NULL, A, (const uint8_t*)A, (const float*)A, A, (const uint8_t*)A, 100,
                                     (const int32_t*)A, 1, 10, (int32_t*)A, A, (size_t)1 << 20, NULL, NULL);
  csa_status s_bad = csa_compress(&bad, A, A, (const float*)A, 8, (const int32_t*)A, (const int32_t*)A,
                                  (const int32_t*)A, 1, NULL, kv, NULL, NULL, NULL);
  csa_status s_align = csa_compress(&p, (const char*)A + 4, A, (const float*)A, 8, (const int32_t*)A,
                                    (const int32_t*)A, (const int32_t*)A, 1, NULL, kv, NULL, NULL, NULL);
  size_t ws = csa_index_topk_workspace_bytes(&p, 1, 32768);
  printf("%d %d %d %zu %s\n", (int)s_null, (int)s_bad, (int)s_align, ws, csa_status_string(CSA_ERR_ALIGN));
  return 0;
}
