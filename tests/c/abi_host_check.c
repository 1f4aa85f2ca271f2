/* A plain C caller of libcalibatt's host entry points (no CUDA calls, no GPU):
 * the header compiles as C, the library links, and the plan builders,
 * balancer, head sharding and small helpers behave as documented.
 * Prints "ok" and returns 0, or names the first failed check. */
#include <math.h>
#include <stdio.h>
#include <stdlib.h>

#include "calibatt.h"

#define CHECK(cond)                                            \
  do {                                                         \
    if (!(cond)) {                                             \
      printf("failed: %s (line %d)\n", #cond, __LINE__);       \
      return 1;                                                \
    }                                                          \
  } while (0)

enum { HEADS = 3, NB = 7, UNITS = HEADS * NB };

int main(void) {
  CHECK(calibatt_version() >= 100);
  CHECK(fabs(calibatt_eps_schedule(0.84, 0.99, 5.0, 0.5, 1.0) - 0.852312749793585) < 1e-15);
  CHECK(calibatt_strerror(0) != NULL);

  int32_t anchors[5];
  CHECK(calibatt_anchor_rows(45, 5, anchors) == CALIBATT_OK);
  CHECK(anchors[0] == 4 && anchors[1] == 13 && anchors[2] == 22 && anchors[3] == 31 && anchors[4] == 40);
  CHECK(calibatt_anchor_rows(4, 5, anchors) == CALIBATT_ERR_ARG);

  /* kept blocks per block-row: head 0 dense, head 1 sparse, head 2 mixed */
  int32_t kept[UNITS], row_ptr[UNITS + 1];
  row_ptr[0] = 0;
  for (int u = 0; u < UNITS; ++u) {
    const int h = u / NB, r = u % NB;
    kept[u] = h == 0 ? NB : (h == 1 ? 1 + (r & 1) : 1 + r);
    row_ptr[u + 1] = row_ptr[u] + kept[u];
  }
  int32_t work[UNITS], n_work = 0;
  CHECK(calibatt_build_plan(row_ptr, HEADS, NB, NULL, work, &n_work) == CALIBATT_OK);
  CHECK(n_work == UNITS);
  int seen[UNITS] = {0};
  for (int i = 0; i < n_work; ++i) {
    CHECK(work[i] >= 0 && work[i] < UNITS && !seen[work[i]]);
    seen[work[i]] = 1;
    if (i > 0) {
      CHECK(work[i] / NB >= work[i - 1] / NB);  /* head by head */
      if (work[i] / NB == work[i - 1] / NB) CHECK(kept[work[i]] <= kept[work[i - 1]]);  /* longest first */
    }
  }

  /* balanced layout for 8 slots: a permutation within each round of 8 */
  int32_t bal[UNITS];
  for (int i = 0; i < UNITS; ++i) bal[i] = work[i];
  CHECK(calibatt_balance_plan(bal, n_work, row_ptr, HEADS, NB, 8) == CALIBATT_OK);
  for (int r = 0; r < UNITS; r += 8) {
    long long a = 0, b = 0;
    for (int i = r; i < r + 8 && i < UNITS; ++i) {
      a += work[i];
      b += bal[i];
    }
    CHECK(a == b);
  }
  CHECK(calibatt_balance_plan(bal, n_work, row_ptr, HEADS, NB, 1) == CALIBATT_ERR_ARG);

  /* two ranks by kept tiles: every head owned, loads add up */
  int32_t owner[HEADS];
  int64_t load[2];
  CHECK(calibatt_shard_heads(row_ptr, HEADS, NB, NULL, 0, 2, 8, 5, 2, owner, load) == CALIBATT_OK);
  CHECK(load[0] + load[1] == row_ptr[UNITS]);
  for (int h = 0; h < HEADS; ++h) CHECK(owner[h] == 0 || owner[h] == 1);

  /* a malformed skip list is refused on the host */
  int32_t col_idx[UNITS * NB];
  for (int u = 0, c = 0; u < UNITS; ++u)
    for (int j = 0; j < kept[u]; ++j) col_idx[c++] = j;
  CHECK(calibatt_validate_csr(row_ptr, col_idx, HEADS, NB, row_ptr[UNITS]) == CALIBATT_OK);
  col_idx[0] = NB;
  CHECK(calibatt_validate_csr(row_ptr, col_idx, HEADS, NB, row_ptr[UNITS]) == CALIBATT_ERR_CSR);

  printf("ok\n");
  return 0;
}
