/* A plain C99 consumer of libsvgear.so: includes only the public header,
 * links only the library, and exercises the calls that need no GPU
 * (version, status strings, workspace sizes, host-side validation).
 * Exit status 0 when every check holds; otherwise prints the failed check. */
#include <stdio.h>
#include <string.h>

#include "svgear.h"

static int failures = 0;

#define CHECK(cond)                                          \
  do {                                                       \
    if (!(cond)) {                                           \
      fprintf(stderr, "check failed: %s (line %d)\n", #cond, __LINE__); \
      ++failures;                                            \
    }                                                        \
  } while (0)

static svgear_params wan_params(void) {
  svgear_params p;
  memset(&p, 0, sizeof p); /* router and budget 0: the method's defaults */
  p.H = 40; p.Nq = 75600; p.Nk = 75600; p.d = 128; p.Cq = 100; p.Ck = 500;
  p.iters = 10; p.rho = 0.15f; p.scale = 0.0f; p.dtype = SVGEAR_BF16;
  return p;
}

int main(void) {
  svgear_params p = wan_params(), bad;
  char dummy[64];
  void* d = dummy + 16 - ((size_t)dummy & 15); /* any 16-byte aligned non-null address */

  CHECK(strstr(svgear_version(), "sm_100a") != NULL);
  CHECK(strcmp(svgear_status_string(SVGEAR_OK), svgear_status_string(SVGEAR_ERR_INVALID)) != 0);
  CHECK(svgear_status_string(12345) != NULL);
  CHECK(svgear_launch_count() == 0);

  /* workspace sizes are host arithmetic */
  CHECK(svgear_workspace_size(&p) > (size_t)3 * 40 * 75600 * 128 * 2);
  CHECK(svgear_block_error_workspace_size(&p) >= (size_t)40 * 100 * 500 * 4);
  CHECK(svgear_hybrid_attn_workspace_size(&p) > 0);
  CHECK(svgear_kmeans_workspace_size(40, 75600, 128, 1000) > 0);
  CHECK(svgear_permute_workspace_size(40, 75600, 500) > 0);
  bad = p; bad.d = 96;
  CHECK(svgear_workspace_size(&bad) == 0);
  bad = p; bad.router = 7;
  CHECK(svgear_workspace_size(&bad) == 0);
  bad = p; bad.budget = 5;
  CHECK(svgear_workspace_size(&bad) == 0);
  p.router = SVGEAR_ROUTE_MASS; p.budget = SVGEAR_BUDGET_GLOBAL;
  CHECK(svgear_workspace_size(&p) > 0);
  p = wan_params();

  /* validation answers before any device work */
  CHECK(svgear_forward(NULL, NULL, NULL, &p, NULL, NULL, NULL, NULL, 0, NULL, NULL) == SVGEAR_ERR_INVALID);
  CHECK(svgear_forward(d, d, d, NULL, NULL, NULL, d, d, 1u << 30, NULL, NULL) == SVGEAR_ERR_INVALID);
  bad = p; bad.rho = 1.5f;
  CHECK(svgear_forward(d, d, d, &bad, NULL, NULL, d, d, 1u << 30, NULL, NULL) == SVGEAR_ERR_INVALID);
  bad = p; bad.dtype = 9;
  CHECK(svgear_forward(d, d, d, &bad, NULL, NULL, d, d, 1u << 30, NULL, NULL) == SVGEAR_ERR_UNSUPPORTED);
  CHECK(svgear_forward(d, d, d, &p, NULL, NULL, d, NULL, 0, NULL, NULL) == SVGEAR_ERR_WORKSPACE);
  CHECK(svgear_route(NULL, NULL, NULL, &p, NULL, NULL, NULL, NULL, NULL) == SVGEAR_ERR_INVALID);
  CHECK(svgear_route_global(d, NULL, d, d, &p, d, d, d, d, NULL) == SVGEAR_ERR_INVALID);
  CHECK(svgear_kmeans(d, SVGEAR_BF16, 1, 10, 64, 0, 1, NULL, d, d, d, d, 1u << 20, NULL) == SVGEAR_ERR_INVALID);
  CHECK(svgear_launch_count() == 0);

  if (failures) {
    fprintf(stderr, "%d check(s) failed\n", failures);
    return 1;
  }
  printf("abi consumer: all checks passed\n");
  return 0;
}
