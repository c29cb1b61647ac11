/* Host-only use of the C ABI from plain C99: the header compiles as C and
 * the library links and answers without a GPU. Prints one line per check;
 * the exit status is the number of failed checks. */
#include <stdio.h>
#include <string.h>

#include "pisa.h"

static int failed = 0;

static void check(int ok, const char* what) {
  printf("%s %s\n", ok ? "ok" : "FAIL", what);
  if (!ok) ++failed;
}

int main(void) {
  check(pisa_version() >= 100, "version");
  check(strcmp(pisa_status_string(PISA_ERR_WORKSPACE), "PISA_ERR_WORKSPACE") == 0, "status string");

  /* N = 1000, C = 64: M_1 = 16, then 8, 4, 2, 1 -> L = 5, R = 31. */
  int32_t L = 0;
  int64_t off[8];
  check(pisa_pyramid_geometry(1000, 64, 2, &L, off) == PISA_OK && L == 5, "geometry levels");
  check(off[0] == 0 && off[1] == 16 && off[2] == 24 && off[3] == 28 && off[4] == 30 && off[5] == 31,
        "geometry offsets");
  check(pisa_pyramid_rows(1000, 64) == 31, "pyramid rows");
  check(pisa_pyramid_geometry(1000, 64, 3, &L, NULL) == PISA_ERR_INVALID_ARGUMENT, "g != 2 rejected");

  pisa_config cfg = {1, 1000, 8, 2, 128, 64, 2, 16, 4, 1, PISA_DTYPE_BF16, 0.0f};
  size_t whole = pisa_select_workspace_bytes(&cfg);
  pisa_query_span all = {0, 1000}, half = {500, 500}, bad = {600, 500};
  check(whole > 0 && pisa_select_span_workspace_bytes(&cfg, &all) == whole, "span {0, N} is the whole call");
  check(pisa_select_span_workspace_bytes(&cfg, &half) < whole, "half span needs less scratch");
  check(pisa_select_span_workspace_bytes(&cfg, &bad) == 0, "span past N has no workspace");

  /* Rejected before anything is enqueued: no device is touched. */
  uint64_t before = pisa_launch_count();
  void* p = (void*)256;
  check(pisa_select_span(&cfg, &bad, p, p, p, p, NULL, p, whole, NULL) == PISA_ERR_INVALID_ARGUMENT,
        "span past N rejected");
  check(pisa_select(&cfg, p, p, p, p, NULL, p, whole - 1, NULL) == PISA_ERR_WORKSPACE, "small workspace rejected");
  cfg.K = 17;
  check(pisa_sparse_attn_fwd(&cfg, p, p, p, p, p, NULL, NULL, 0, NULL) == PISA_ERR_UNSUPPORTED, "K = 17 unsupported");
  check(pisa_launch_count() == before, "nothing launched");

  /* An empty timing window needs no device and records nothing. */
  const char* names[4];
  double ms[4];
  int launches[4];
  check(pisa_timing_start() == PISA_OK, "timing start");
  check(pisa_timing_stop(4, names, ms, launches) == 0, "empty timing window");
  return failed;
}
