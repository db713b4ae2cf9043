/* Host-only check of the C ABI from plain C: the header compiles as C11, the
 * library links by its extern "C" names, and the planning calls that touch no
 * device behave as the header states.  Exit status 0 on success; prints
 * "abi ok". */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "shampoo4.h"

static int failures = 0;
#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #cond); \
      ++failures;                                                     \
    }                                                                 \
  } while (0)

static int ceil_div(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }

int main(void) {
  /* A 1100 x 700 weight, a 64 x 147 one and a 4 x 4 one, tiles of 512. */
  const shampoo4_param params[3] = {{1100, 700}, {64, 147}, {4, 4}};
  shampoo4_config cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.beta = 0.95f;
  cfg.eps = 1e-6f;
  cfg.max_block = 512;
  cfg.quant_block = 64;
  cfg.bjorck_iters = 5;
  cfg.precision = SHAMPOO4_PREC_TF32;

  shampoo4_handle h = NULL;
  CHECK(shampoo4_init(&cfg, params, 3, &h) == SHAMPOO4_OK && h != NULL);
  if (!h) return 1;

  int32_t nblocks = 0, nfactors = 0;
  CHECK(shampoo4_counts(h, &nblocks, &nfactors) == SHAMPOO4_OK);
  const int want_blocks = ceil_div(1100, 512) * ceil_div(700, 512) + 1 + 1;
  CHECK(nblocks == want_blocks && nfactors == 2 * want_blocks);

  /* tiles in order: parameter, row chunk, column chunk; ragged last chunks */
  int32_t p, m, n;
  int64_t r0, c0;
  CHECK(shampoo4_block_info(h, 0, &p, &r0, &c0, &m, &n) == SHAMPOO4_OK);
  CHECK(p == 0 && r0 == 0 && c0 == 0 && m == 512 && n == 512);
  CHECK(shampoo4_block_info(h, 5, &p, &r0, &c0, &m, &n) == SHAMPOO4_OK);
  CHECK(p == 0 && r0 == 1024 && c0 == 512 && m == 76 && n == 188);
  CHECK(shampoo4_block_info(h, 6, &p, &r0, &c0, &m, &n) == SHAMPOO4_OK);
  CHECK(p == 1 && m == 64 && n == 147);
  CHECK(shampoo4_block_info(h, nblocks, &p, &r0, &c0, &m, &n) == SHAMPOO4_ERR_INVALID_ARG);

  size_t state = 0, ws = 0;
  CHECK(shampoo4_sizes(h, &state, &ws) == SHAMPOO4_OK && state > 0 && ws > 0);
  for (int32_t f = 0; f < nfactors; ++f) {
    size_t oS, oc, os, ol;
    int32_t d;
    CHECK(shampoo4_factor_layout(h, f, &oS, &oc, &os, &ol, &d) == SHAMPOO4_OK);
    const size_t dd = (size_t)d * (size_t)d;
    CHECK(oS % 256 == 0 && oc % 256 == 0 && os % 256 == 0 && ol % 256 == 0);
    CHECK(oS + 4 * dd <= state && oc + (dd + 1) / 2 <= state && ol + 4 * (size_t)d <= state);
  }

  /* grafting state: Adam moments, 8 bytes per parameter element (plus
     alignment); SGD needs none */
  size_t gb = 1;
  CHECK(shampoo4_graft_state_bytes(h, SHAMPOO4_GRAFT_SGD, &gb) == SHAMPOO4_OK && gb == 0);
  CHECK(shampoo4_graft_state_bytes(h, SHAMPOO4_GRAFT_ADAM, &gb) == SHAMPOO4_OK);
  CHECK(gb >= 8u * (1100u * 700u + 64u * 147u + 16u) && gb % 256 == 0);

  /* one rank: it owns every factor and one span */
  int32_t owner = -1;
  CHECK(shampoo4_factor_owner(h, 0, &owner) == SHAMPOO4_OK && owner == 0);
  size_t soff = 1, sbytes = 0;
  CHECK(shampoo4_owner_span(h, 0, &soff, &sbytes) == SHAMPOO4_OK && soff == 0 && sbytes > 0);
  CHECK(shampoo4_owner_span(h, 1, &soff, &sbytes) == SHAMPOO4_ERR_INVALID_ARG);

  /* debug capture: two fp32 d x d matrices per factor, 256-byte aligned,
     disjoint; a misaligned buffer is refused */
  size_t dbytes = 0;
  CHECK(shampoo4_debug_capture_bytes(h, &dbytes) == SHAMPOO4_OK && dbytes % 256 == 0);
  for (int32_t f = 0; f < nfactors; ++f) {
    size_t ou = 1, oq = 1;
    int32_t d;
    CHECK(shampoo4_factor_layout(h, f, NULL, NULL, NULL, NULL, &d) == SHAMPOO4_OK);
    CHECK(shampoo4_debug_capture_layout(h, f, &ou, &oq) == SHAMPOO4_OK);
    CHECK(ou % 256 == 0 && oq % 256 == 0 && ou + 4 * (size_t)d * (size_t)d <= oq);
    CHECK(oq + 4 * (size_t)d * (size_t)d <= dbytes);
  }
  CHECK(shampoo4_debug_capture(h, (void*)(uintptr_t)0x1010) == SHAMPOO4_ERR_INVALID_ARG);

  /* calls that need bound buffers are refused before touching a device */
  CHECK(shampoo4_refresh_roots(h, NULL) == SHAMPOO4_ERR_NOT_READY);
  shampoo4_destroy(h);

  /* bad configurations are refused at init */
  shampoo4_config bad = cfg;
  bad.quant_block = 32;
  h = NULL;
  CHECK(shampoo4_init(&bad, params, 3, &h) == SHAMPOO4_ERR_INVALID_ARG && h == NULL);
  bad = cfg;
  bad.refresh_world = 2;
  bad.refresh_rank = 2;
  CHECK(shampoo4_init(&bad, params, 3, &h) == SHAMPOO4_ERR_INVALID_ARG);

  /* two ranks: every factor has one owner, spans are disjoint */
  shampoo4_handle r0h = NULL, r1h = NULL;
  shampoo4_config c2 = cfg;
  c2.refresh_world = 2;
  c2.refresh_rank = 0;
  CHECK(shampoo4_init(&c2, params, 3, &r0h) == SHAMPOO4_OK);
  c2.refresh_rank = 1;
  CHECK(shampoo4_init(&c2, params, 3, &r1h) == SHAMPOO4_OK);
  if (r0h && r1h) {
    size_t a0, b0, a1, b1, x0, y0, x1, y1;
    CHECK(shampoo4_owner_span(r0h, 0, &a0, &b0) == SHAMPOO4_OK && shampoo4_owner_span(r0h, 1, &a1, &b1) == SHAMPOO4_OK);
    CHECK(shampoo4_owner_span(r1h, 0, &x0, &y0) == SHAMPOO4_OK && shampoo4_owner_span(r1h, 1, &x1, &y1) == SHAMPOO4_OK);
    CHECK(a0 == x0 && b0 == y0 && a1 == x1 && b1 == y1);
    CHECK(a0 + b0 <= a1 || a1 + b1 <= a0);
    int owned[2] = {0, 0};
    for (int32_t f = 0; f < nfactors; ++f) {
      int32_t o0 = -1, o1 = -1;
      CHECK(shampoo4_factor_owner(r0h, f, &o0) == SHAMPOO4_OK && shampoo4_factor_owner(r1h, f, &o1) == SHAMPOO4_OK);
      CHECK(o0 == o1 && (o0 == 0 || o0 == 1));
      if (o0 == 0 || o0 == 1) ++owned[o0];
    }
    CHECK(owned[0] > 0 && owned[1] > 0);
  }
  shampoo4_destroy(r0h);
  shampoo4_destroy(r1h);

  CHECK(strlen(shampoo4_status_string(SHAMPOO4_ERR_NOT_READY)) > 0);
  CHECK(strcmp(shampoo4_stage_name(0), "stats_scan") == 0);
  CHECK(strcmp(shampoo4_stage_name(SHAMPOO4_STAGE_COUNT), "unknown") == 0);
  if (failures) {
    fprintf(stderr, "%d check(s) failed\n", failures);
    return 1;
  }
  printf("abi ok\n");
  return 0;
}
