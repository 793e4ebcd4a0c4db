/*
 * A C99 program against the library's C ABI (include/calibatt.h).  It checks
 * that the header compiles as plain C with strict warnings, that every call
 * used here links against libcalibatt.so, and that the calls answer on the
 * host: each one is host arithmetic or is refused by its argument checks
 * before any CUDA call, so no GPU is needed.  Exit status 0 and "c abi ok" on
 * success; each failed check is printed to stderr.
 */
#include <stdio.h>
#include <string.h>

#include "calibatt.h"

static int fails = 0;

#define CHECK(cond)                                                      \
  do {                                                                   \
    if (!(cond)) {                                                       \
      fprintf(stderr, "FAIL %s:%d: %s\n", __FILE__, __LINE__, #cond);    \
      ++fails;                                                           \
    }                                                                    \
  } while (0)

int main(void) {
  int32_t mv = -1, k = -1;
  int32_t anchors[5], nearest[30];
  int nq = 0, npq = 0;
  size_t bytes = 0;
  int64_t csr = 0, pool = 0;
  uint64_t old_limit;
  calibatt_blocklist bl;

  CHECK(calibatt_version() == 10000);

  /* agreement threshold ceil(rho I) and top-k count ceil(frac nkb) */
  CHECK(calibatt_min_votes(0.5, 8, &mv) == CALIBATT_OK && mv == 4);
  CHECK(calibatt_min_votes(0.3, 10, &mv) == CALIBATT_OK && mv == 3);
  CHECK(calibatt_topk_count(0.25, 256, &k) == CALIBATT_OK && k == 64);
  CHECK(calibatt_topk_count(0.2, 591, &k) == CALIBATT_OK && k == 119);
  CHECK(calibatt_topk_count(0.0, 10, &k) == CALIBATT_E_INVALID);

  /* 5 anchor rows of 30, evenly spaced and centred: rows 3, 9, 15, 21, 27;
   * row 0 takes row 3, row 6 (equidistant from 3 and 9) the lower one */
  CHECK(calibatt_anchor_rows(30, 5, anchors, nearest) == CALIBATT_OK);
  CHECK(anchors[0] == 3 && anchors[1] == 9 && anchors[2] == 15 && anchors[3] == 21 && anchors[4] == 27);
  CHECK(nearest[0] == 3 && nearest[6] == 3 && nearest[7] == 9 && nearest[29] == 27);
  CHECK(calibatt_anchor_rows(30, 31, anchors, nearest) == CALIBATT_E_INVALID);

  /* 21 frames x 5 anchor rows x 52 columns = 5 460 gathered queries, padded to 5 504 */
  CHECK(calibatt_anchor_plan_size(21, 30, 52, 5, &nq, &npq) == CALIBATT_OK && nq == 5460 && npq == 5504);

  CHECK(calibatt_calibrate_workspace_size(40, 32760, 32768, 128, 128, 128, &bytes) == CALIBATT_OK && bytes > 0);
  CHECK(calibatt_compile_workspace_size(4800, 256, 256, &bytes) == CALIBATT_OK && bytes > 0);
  CHECK(calibatt_blocklist_bytes(2, 8, 10, 3, 4, &csr, &pool) == CALIBATT_OK);
  CHECK(csr == 17 * 8 + 10 * 2 && pool == 16 * 8 + 4 * 4 + 4 * 2);

  /* refused on the host, with a message */
  memset(&bl, 0, sizeof bl);
  CHECK(calibatt_sparse_attn_fwd(NULL, NULL, NULL, NULL, NULL, 1, 1, 128, 128, 128, CALIBATT_BF16, 0.1f, &bl, 0,
                                 NULL, NULL) == CALIBATT_E_INVALID);
  CHECK(strstr(calibatt_last_error(), "non-NULL") != NULL);
  CHECK(calibatt_selftest_wait_timeout(0, NULL, NULL) == CALIBATT_E_INVALID);

  old_limit = calibatt_get_spin_limit_ns();
  calibatt_set_spin_limit_ns(12345);
  CHECK(calibatt_get_spin_limit_ns() == 12345);
  calibatt_set_spin_limit_ns(old_limit);

  if (fails) return 1;
  printf("c abi ok\n");
  return 0;
}
