/* Plain-C client of libetp: the boundary needs nothing beyond a C compiler and the header.
 * Exercises the host-only calls (no GPU): handle lifecycle, info, path list, workspace query and
 * the status strings; prints one line per check and returns non-zero on the first mismatch. */
#include <stdio.h>
#include <string.h>

#include "etp.h"

static int fail(const char* what) {
  printf("FAIL %s: %s\n", what, etp_last_error());
  return 1;
}

int main(void) {
  etp_handle h = NULL;
  etp_info_t info;
  int paths[3 * 64];
  if (etp_create("64x0e+64x1o+64x2e", 2, "64x0e+64x1o+64x2e", 8, 5.0f, &h) != ETP_OK) return fail("create uniform");
  if (etp_get_info(h, &info) != ETP_OK) return fail("info uniform");
  if (info.general != 0 || info.n_paths != 11 || info.dim_in != 576 || info.weight_numel != 8 * 11 * 64)
    return fail("uniform info values");
  if (etp_get_paths(h, paths, 64) != ETP_OK) return fail("paths uniform");
  if (paths[0] != 0 || paths[1] != 0 || paths[2] != 0) return fail("first path (0,0,0)");
  if (etp_workspace_bytes(h, 1000, 89156) < 2 * 4 * 89156) return fail("workspace size");
  {
    int code = -1;
    int* word = etp_status_word(h);
    if (!word || *word != 0) return fail("status word starts clear");
    *word = 9;
    if (etp_get_status(h, NULL, &code) != ETP_ERR_CUDA || code != 9 || *word != 0) return fail("status read");
    if (etp_get_status(h, NULL, &code) != ETP_OK || code != 0) return fail("status cleared");
  }
  etp_destroy(h);
  printf("ok uniform: %d paths, dim %d, weights %d\n", info.n_paths, info.dim_in, info.weight_numel);

  if (etp_create("128x0e+64x1o+32x2e+32x3o", 3, "128x0e+64x1o+32x2e+32x3o", 8, 5.0f, &h) != ETP_OK)
    return fail("create general");
  if (etp_get_info(h, &info) != ETP_OK) return fail("info general");
  if (info.general != 1 || info.channels != 0 || info.dim_in != 128 + 192 + 160 + 224) return fail("general info");
  if (etp_get_paths(h, paths, 1) != ETP_ERR_CAPACITY) return fail("capacity check");
  etp_destroy(h);
  printf("ok general: %d paths, dim %d, weights %d\n", info.n_paths, info.dim_in, info.weight_numel);

  if (etp_create("64x0e+64x1q", 1, "64x0e", 8, 5.0f, &h) != ETP_ERR_IRREPS || h != NULL) return fail("malformed");
  if (strcmp(etp_status_string(ETP_ERR_IRREPS), "malformed irreps string") != 0) return fail("status string");
  printf("ok errors: %s\n", etp_last_error());
  return 0;
}
