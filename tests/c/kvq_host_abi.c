/* Plain C use of the libkvq C ABI, host-only calls (no GPU needed): the
 * library version, sizes, a codebook, a plan built from energies and its
 * check. Compiled and run by tests/test_c_abi.py; prints one line per fact. */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "kvq.h"

int main(void) {
  kvq_cfg cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.head_dim = 128;
  cfg.n_kv_heads = 2;
  cfg.bits_k = 3;
  cfg.bits_v = 3;
  cfg.b_max = 8;
  cfg.alloc_mode = KVQ_ALLOC_GREEDY;
  cfg.v_seed = 7;

  printf("version %s\n", kvq_version());
  printf("plan_bytes %zu\n", kvq_plan_bytes());
  printf("tile_bytes %zu\n", kvq_tile_bytes(&cfg));
  printf("cache_bytes_128k %zu\n", kvq_cache_bytes(&cfg, 131072));
  printf("page_bytes_16 %zu\n", kvq_page_bytes(&cfg, 16));

  float c[8], t[7];
  double d = 0.0;
  if (kvq_codebook(3, c, t, &d) != KVQ_OK) return 1;
  printf("codebook3 %.6f %.6f %.6f\n", c[0], t[3], d);

  double E[2 * 64];
  for (int h = 0; h < 2; ++h)
    for (int j = 0; j < 64; ++j) E[h * 64 + j] = 1.0 / (1.0 + j + h);
  unsigned char* plans = (unsigned char*)calloc(2, kvq_plan_bytes());
  if (kvq_plan_build(&cfg, 0, E, 2, plans) != KVQ_OK) return 2;
  for (int h = 0; h < 2; ++h)
    if (kvq_plan_check(&cfg, plans + h * kvq_plan_bytes()) != KVQ_OK) return 3;
  int sum = 0;
  for (int j = 0; j < 64; ++j) sum += plans[544 + j]; /* width[64] at byte 544 */
  printf("plan_width_sum %d\n", sum);
  plans[544] = 9; /* a width past 8: the check refuses it */
  const int rc = kvq_plan_check(&cfg, plans);
  printf("corrupt_plan_check %d %s\n", rc, kvq_last_error());
  cfg.head_dim = 64;
  printf("head_dim_64 %d\n", kvq_plan_build(&cfg, 0, E, 1, plans));
  free(plans);
  return 0;
}
