/*
 * Plain C99 use of the library's C ABI (include/jl_api.h): the header compiles
 * as strict C, the library links with nothing but its path, and the host-only
 * entry points answer without a GPU.  Exit status 0 on success, otherwise the
 * number of the first failed check.
 */
#include <stdint.h>
#include <stdio.h>

#include "jl_api.h"

int main(void) {
  int64_t G = 0;
  int32_t q[16], k[16];
  int64_t c[4];
  int i;
  /* G = max(1, ceil(L / w_pretrained)) */
  if (jl_group_size(131072, 32768, &G) != JL_OK || G != 4) return 1;
  if (jl_group_size(16, 0, &G) != JL_ERR_INVALID_ARG) return 2;
  /* L 16, w_pretrained 4: G 4, f(j) = j / 4; Self-Extend shift w0 - w0 / G = 4 - 1 */
  if (jl_remote_positions(16, 4, 4, JL_QSHIFT_SELF_EXTEND, q, k) != JL_OK) return 3;
  for (i = 0; i < 16; ++i)
    if (k[i] != i / 4 || q[i] != i / 4 + 3) return 4;
  /* L 512, w0 32: seven 128 x 128 tiles straddle the band edge, three are remote only */
  if (jl_prefill_tile_classes(512, 32, 128, c) != JL_OK) return 5;
  if (c[0] != 0 || c[1] != 7 || c[2] != 3 || c[3] != 17) return 6;
  /* argument checks come before any pointer is touched or kernel launched */
  if (jl_bifocal_prefill(NULL, NULL, NULL, NULL, NULL, 1, 256, 4, 2, 96, 16, 64, 1e4, 0.f, JL_QSHIFT_SELF_EXTEND,
                         NULL, 0, NULL, NULL) != JL_ERR_UNSUPPORTED)
    return 7;
  if (jl_bifocal_prefill(NULL, NULL, NULL, NULL, NULL, 1, 256, 4, 2, 128, 16, 64, 1e4, 0.f, JL_QSHIFT_SELF_EXTEND,
                         NULL, 0, NULL, NULL) != JL_ERR_INVALID_ARG)
    return 8;
  if (jl_prefill_workspace_bytes(1, 512, 2, 1, 64) == 0 || jl_prefill_workspace_bytes(0, 512, 2, 1, 64) != 0) return 9;
  printf("%s\n", jl_status_string(JL_ERR_ALIGNMENT));
  return 0;
}
