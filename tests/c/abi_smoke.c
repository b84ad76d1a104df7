/* Plain-C client of libwave.so (no Python, no CUDA headers): the header must be
 * valid C99 and the host-side calls must work through the C ABI alone.
 * Prints one line per check; exits non-zero on the first failure. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "wave.h"

#define CHECK(cond, what)                                                   \
  do {                                                                      \
    if (!(cond)) {                                                          \
      fprintf(stderr, "FAIL %s: %s\n", what, wave_last_error_detail());     \
      return 1;                                                             \
    }                                                                       \
    printf("ok %s\n", what);                                                \
  } while (0)

int main(void) {
  /* Progressive schedule of 3 chunks, 2 levels: 4 rounds. */
  wave_node nodes[64];
  int32_t offs[65], n_nodes = 0, n_rounds = 0;
  int rc = wave_schedule(3, 2, WAVE_POLICY_PROGRESSIVE, 0, nodes, 64, offs, 65, &n_nodes, &n_rounds);
  CHECK(rc == WAVE_OK && n_rounds == 4, "schedule B=3 K=2 progressive has 4 rounds");
  CHECK(offs[0] == 0 && offs[n_rounds] == n_nodes, "round offsets span the node list");
  CHECK(nodes[0].chunk == 0 && nodes[0].level == 2, "round 0 is (0, 2)");

  /* Too-small capacity reports the sizes needed. */
  int32_t need_nodes = 0, need_rounds = 0;
  rc = wave_schedule(3, 2, WAVE_POLICY_PROGRESSIVE, 0, nodes, 1, offs, 65, &need_nodes, &need_rounds);
  CHECK(rc == WAVE_ERR_CAPACITY && need_nodes == n_nodes, "capacity error gives the size needed");

  /* Host-only cache handle: tables without a device. */
  wave_kv_config cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.heads = 2;
  cfg.head_dim = 64;
  cfg.tokens_per_chunk = 200;
  cfg.num_levels = 2;
  cfg.pool = NULL;
  int64_t page_bytes = 2LL * 2 * 128 * 64 * 2;
  cfg.pool_bytes = (uint64_t)(4096 + 8 * page_bytes);
  wave_kv* kv = NULL;
  CHECK(wave_kv_create(&cfg, &kv) == WAVE_OK && kv != NULL, "host-only handle");
  int32_t free_pages = 0;
  CHECK(wave_kv_free_pages(kv, &free_pages) == WAVE_OK && free_pages == 8, "8 free pages");
  CHECK(wave_kv_alloc(kv, 0, 0, 200) == WAVE_OK, "alloc (0, 0)");
  CHECK(wave_kv_alloc(kv, 1, 1, 200) == WAVE_OK, "alloc (1, 1)");
  CHECK(wave_kv_alloc(kv, 1, 1, 200) == WAVE_ERR_EXISTS, "second alloc of (1, 1) is EXISTS");

  /* (1, 1) under clean reads E(0, 0) then itself: pages 0, 1 then 2, 3. */
  wave_node act[1] = {{1, 1}};
  int32_t rows[16], roffs[2], n_rows = 0;
  rc = wave_gather_table(kv, act, 1, WAVE_POLICY_CLEAN, rows, roffs, 8, &n_rows);
  CHECK(rc == WAVE_OK && n_rows == 4, "gather table of (1, 1) has 4 pages");
  CHECK(rows[0] == 0 && rows[1] == 128 && rows[2] == 1 && rows[3] == 72, "history pages 0, 1");
  CHECK(rows[4] == 2 && rows[5] == 128 && rows[6] == 3 && rows[7] == 72, "own pages 2, 3");
  rc = wave_gather_table(kv, act, 1, WAVE_POLICY_SAME, rows, roffs, 8, &n_rows);
  CHECK(rc == WAVE_ERR_MISSING_KV, "same-level needs E(0, 1): MISSING_KV");

  int32_t own[4], n_own = 0;
  CHECK(wave_kv_entry_pages(kv, 1, 1, own, 4, &n_own) == WAVE_OK && n_own == 2 && own[0] == 2 &&
            own[1] == 3, "entry pages of (1, 1) are 2, 3");
  CHECK(wave_kv_set_wait_limit(kv, 5000) == WAVE_OK, "wait limit set");
  CHECK(wave_kv_release(kv, 0, 0) == WAVE_OK, "release (0, 0)");
  CHECK(wave_kv_free_pages(kv, &free_pages) == WAVE_OK && free_pages == 6, "6 free pages");

  /* Wave Parallelism, progressive, B = 3, K = 2 on 3 ranks: round 2 runs
   * (0, 0), (1, 1), (2, 2); E(0, 0) goes from rank 0 to ranks 1 and 2. */
  wave_transfer tr[8];
  int32_t n_tr = 0;
  rc = wave_wp_transfers(3, 2, WAVE_POLICY_PROGRESSIVE, 0, 3, 2, tr, 8, &n_tr);
  CHECK(rc == WAVE_OK && n_tr >= 2 && tr[0].chunk == 0 && tr[0].level == 0 && tr[0].src == 0,
        "round 2 pushes E(0, 0) from rank 0");
  int all_one_way = 1;
  for (int32_t i = 0; i < n_tr; ++i) all_one_way &= tr[i].dst > tr[i].src;
  CHECK(all_one_way, "progressive pushes go from a cleaner to a noisier rank");
  CHECK(strlen(wave_strerror(WAVE_ERR_NO_PAGES)) > 0, "strerror names codes");
  CHECK(wave_kv_destroy(kv) == WAVE_OK, "destroy");
  return 0;
}
