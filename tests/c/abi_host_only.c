/* Plain-C client of the library's C ABI (no GPU needed): checks that
 * include/ringattn.h and include/ringattn_debug.h compile as C99 and that the
 * host-only entry points answer from C.  Built and run by tests/test_abi.py. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "ringattn.h"
#include "ringattn_debug.h"

int main(void) {
  /* causal visible pairs: S (S + 1) / 2 per (b, h) */
  const int64_t S = 1000;
  int64_t n = ra_count_visible_pairs(2, S, 3, 1, NULL, NULL);
  if (n != 2 * 3 * S * (S + 1) / 2) { printf("count %lld\n", (long long)n); return 1; }
  /* ring order of the tiles seen by query rows [0, 127] of a 4-block ring */
  ra_params p;
  memset(&p, 0, sizeof p);
  p.query_chunk_size = 256;
  p.key_chunk_size = 256;
  p.causal_block_size = 0;
  p.ring_size = 4;
  int32_t tiles[64];
  int64_t m = ra_ring_schedule(1024, &p, 0, 127, NULL, NULL, tiles, 64);
  if (m != 8) { printf("schedule length %lld\n", (long long)m); return 2; }
  /* block 0 first (its own keys), then blocks 3, 2, 1 (step t visits block (0 - t) mod 4) */
  const int32_t want[8] = {0, 1, 6, 7, 4, 5, 2, 3};
  for (int i = 0; i < 8; ++i)
    if (tiles[i] != want[i]) { printf("tile %d: %d\n", i, tiles[i]); return 3; }
  if (strcmp(ra_strerror(RA_OK), "ok") != 0) return 4;
  if (ra_forward(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) != RA_ERR_NULL) return 5;
  if (ra_train_step_host(NULL, NULL, NULL, &p, 1, NULL, 0, NULL, NULL, NULL) != RA_ERR_NULL) return 6;
  printf("ok\n");
  return 0;
}
