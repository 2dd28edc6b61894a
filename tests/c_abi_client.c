/*
 * A plain C99 client of include/sla.h: the header compiles as C with -pedantic
 * and the library links and answers without Python, torch or a GPU. Only
 * host-side entry points are called (validation, sizes, stage names, the
 * Hilbert order, argument checks that return before any launch).
 * Prints "ok" and exits 0, or names the first failed check and exits 1.
 */
#include <stdio.h>
#include <string.h>

#include "sla.h"

#define CHECK(cond)                                          \
  do {                                                       \
    if (!(cond)) {                                           \
      fprintf(stderr, "failed: %s (line %d)\n", #cond, __LINE__); \
      return 1;                                              \
    }                                                        \
  } while (0)

static sla_config wan_like(void) {
  /* the Wan2.1-1.3B-shaped layer: 12 heads, 32760 valid tokens padded to 32768 */
  sla_config c;
  memset(&c, 0, sizeof(c));
  c.B = 1;
  c.H = 12;
  c.H_kv = 12;
  c.N = 32768;
  c.N_valid = 32760;
  c.d = 128;
  c.block = 64;
  c.mode = SLA_MODE_THREEWAY;
  c.k_h = 26;
  c.k_l = 51;
  c.has_proj = 1;
  return c;
}

int main(void) {
  sla_config c = wan_like();
  sla_config bad = c;
  int32_t order[2 * 3 * 5];
  int seen[2 * 3 * 5];
  int i, n_stages;
  size_t ws;

  CHECK(sla_version() != NULL && strlen(sla_version()) > 0);
  CHECK(sla_validate_config(&c) == SLA_OK);
  ws = sla_workspace_bytes(&c);
  CHECK(ws > 0);

  n_stages = sla_num_stages(&c);
  CHECK(n_stages == 6);
  CHECK(strcmp(sla_stage_name(&c, 0), "pool") == 0);
  CHECK(sla_stage_name(&c, n_stages) == NULL);

  bad.N = 1000; /* not a multiple of the block */
  CHECK(sla_validate_config(&bad) == SLA_ERR_INVALID_ARG);
  CHECK(sla_workspace_bytes(&bad) == 0);
  bad = c;
  bad.d = 96;
  CHECK(sla_validate_config(&bad) == SLA_ERR_UNSUPPORTED);

  /* argument checks return before any launch */
  CHECK(sla_forward(NULL, NULL, NULL, NULL, NULL, &c, NULL, NULL, NULL, 0, NULL) == SLA_ERR_INVALID_ARG);
  CHECK(sla_forward_host_device_bytes(&c, 12) > ws);
  CHECK(sla_forward_host_device_bytes(&c, 5) == 0);
  CHECK(sla_status_string(SLA_ERR_WORKSPACE) != NULL);

  /* the Hilbert order of a 2 x 3 x 5 grid is a permutation of the raster indices */
  CHECK(sla_hilbert_order(2, 3, 5, order) == SLA_OK);
  memset(seen, 0, sizeof(seen));
  for (i = 0; i < 30; ++i) {
    CHECK(order[i] >= 0 && order[i] < 30);
    seen[order[i]] += 1;
  }
  for (i = 0; i < 30; ++i) CHECK(seen[i] == 1);
  CHECK(sla_hilbert_order(0, 3, 5, order) == SLA_ERR_INVALID_ARG);

  printf("ok\n");
  return 0;
}
