/* A plain C99 caller of libwtconv.so: includes only wtconv.h, links only the
 * library, and makes calls that the library answers on the host before any
 * launch (sizes, launch counts, status strings, argument errors), so it runs
 * on a machine without a GPU.  It prints one "name value" line per result;
 * the test that builds it compares them with the same calls made through
 * the Python binding. */
#include <stdio.h>
#include <stdint.h>

#include "wtconv.h"

#define FAKE ((void*)(uintptr_t)0x10000) /* 16-byte aligned, never dereferenced */

int main(void) {
  const wtconv_desc d = {2, 3, 16, 16, 5, 2, WTCONV_F32};
  const wtconv_desc even_k = {2, 3, 16, 16, 4, 2, WTCONV_F32};
  const wtconv_desc ragged = {2, 3, 16, 10, 5, 2, WTCONV_BF16};
  /* one group of partial sums (C * (k*k*(1+4L)+1) floats) over the
   * no-allocation array */
  const int V = 25 * (1 + 4 * 2) + 1;
  const wtconv_desc huge_c = {1, (int)(WTCONV_NOALLOC_SCRATCH_BYTES / (V * 4)) + 1, 16, 16, 5, 2, WTCONV_F32};
  const float* fp = (const float*)FAKE;
  float* op = (float*)FAKE;
  int op_code;

  for (op_code = 0; op_code <= 3; ++op_code)
    printf("ws_%d %zu\n", op_code, wtconv_workspace_size(&d, op_code));
  printf("ws_ragged_2 %zu\n", wtconv_workspace_size(&ragged, WTCONV_OP_BACKWARD_WEIGHT));
  printf("ws_even_k %zu\n", wtconv_workspace_size(&even_k, WTCONV_OP_FORWARD));
  printf("folded %zu\n", wtconv_folded_size(&d));
  for (op_code = 0; op_code <= 5; ++op_code)
    printf("launches_%d %d\n", op_code, wtconv_kernel_launches(&d, op_code));

  printf("fwd_null_x %d\n",
         (int)wtconv_forward(&d, NULL, fp, fp, fp, fp, fp, FAKE, FAKE, (size_t)1 << 30, NULL));
  printf("fwd_even_k %d\n",
         (int)wtconv_forward(&even_k, FAKE, fp, fp, fp, fp, fp, FAKE, FAKE, (size_t)1 << 30, NULL));
  printf("fwd_small_ws %d\n",
         (int)wtconv_forward(&d, FAKE, fp, fp, fp, fp, fp, FAKE, FAKE, 16, NULL));
  printf("bwd_data_misaligned %d\n",
         (int)wtconv_backward_data(&d, (const char*)FAKE + 4, fp, fp, fp, fp, FAKE, FAKE, (size_t)1 << 30, NULL));
  printf("noalloc_ragged %d\n",
         (int)wtconv_backward_weight_noalloc(&ragged, FAKE, FAKE, fp, fp, fp, fp, fp, op, op, op, op, op, NULL));
  printf("noalloc_huge_c %d\n",
         (int)wtconv_backward_weight_noalloc(&huge_c, FAKE, FAKE, fp, fp, fp, fp, fp, op, op, op, op, op, NULL));
  printf("scratch_bytes %zu\n", wtconv_noalloc_scratch_bytes());
  printf("scratch_macro %zu\n", (size_t)WTCONV_NOALLOC_SCRATCH_BYTES);
  printf("status_string_ok %s\n", wtconv_status_string(WTCONV_OK) ? "set" : "null");
  printf("status_string_limit %s\n", wtconv_status_string(WTCONV_ERR_SCRATCH_LIMIT) ? "set" : "null");
  return 0;
}
