/* Calls the library from plain C (no CUDA headers, no GPU work): the header compiles as C and
 * the host-side entry points answer as documented.  Built and run by tests/test_c_abi.py. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "mlra.h"

int main(void) {
  if (mlra_version() <= 0) { printf("bad version\n"); return 1; }
  const char* s = mlra_status_string(MLRA_ERR_INVALID_ARG);
  if (!s || !strstr(s, "INVALID_ARG")) { printf("bad status string\n"); return 1; }
  /* sizes without a device: an explicit range count skips the SM query */
  mlra_dims d;
  memset(&d, 0, sizeof d);
  d.batch = 2; d.heads = 64; d.num_branches = 4; d.d_latent = 512; d.d_rope = 64;
  d.max_seq_len = 1024; d.cache_rows = 2048; d.c_row_stride = 512; d.kr_row_stride = 64;
  d.dtype = MLRA_BF16; d.out_mode = MLRA_OUT_BRANCHES; d.num_ranges = 8;
  size_t bytes = 0;
  if (mlra_workspace_size(&d, &bytes) != MLRA_OK || bytes == 0) { printf("workspace\n"); return 1; }
  size_t bytes2 = 0;
  if (mlra_workspace_size_multi(&d, 2, &bytes2) != MLRA_OK || bytes2 <= bytes) {
    printf("workspace multi\n");
    return 1;
  }
  d.heads = 129;
  if (mlra_workspace_size(&d, &bytes) != MLRA_ERR_UNSUPPORTED) { printf("heads\n"); return 1; }
  /* the split plan on the host: 3 sequences of 5, 0 and 7 tiles over 4 ranges */
  const int32_t tiles[3] = {5, 0, 7};
  int32_t first[4], parts[3];
  if (mlra_plan_host(tiles, 3, 4, 0, first, parts) != MLRA_OK) { printf("plan\n"); return 1; }
  if (parts[1] != 0 || parts[0] < 1 || parts[2] < 1) { printf("plan parts\n"); return 1; }
  if (mlra_decode(NULL, NULL, NULL, NULL, NULL, NULL, 4, NULL, NULL, NULL, &d, NULL, 0, NULL) !=
      MLRA_ERR_INVALID_ARG) {
    printf("decode args\n");
    return 1;
  }
  printf("ok %zu %zu\n", bytes2, bytes);
  return 0;
}
