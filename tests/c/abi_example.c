/* A plain C99 caller of libcce.so: only include/cce.h and the shared library, no torch. It makes
 * the calls that need no GPU (sizes, argument validation, status strings) and prints what the test
 * checks. */
#include <stdio.h>
#include <stdint.h>

#include "cce.h"

int main(void) {
  cce_problem p = {4096, 4096, 128256, -100, CCE_REDUCTION_MEAN, 0, 0.0f, 0.0f};
  int32_t rows = 0, cols = 0;
  cce_backward_tile_shape(&rows, &cols);
  printf("version %d\n", (int)cce_version());
  printf("tile %d %d\n", (int)rows, (int)cols);
  printf("tile_max_len %lld\n", (long long)cce_tile_max_len(&p));
  printf("fwd_ws %zu\n", cce_forward_workspace_size(&p));
  printf("bwd_ws %zu\n", cce_backward_workspace_size(&p, 0));
  cce_problem bad = p;
  bad.D = 7; /* not a multiple of 8 */
  cce_status st = cce_forward(&bad, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL);
  printf("bad_status %d %s\n", (int)st, cce_status_string(st));
  printf("message %s\n", cce_last_error_message());
  return 0;
}
