/* Plain C use of the library's ABI on the host: a host-only plan (no device),
 * its geometry, KV-tile list of one query tile, launch counts, workspace sizes
 * and two rejected problems.  Prints one "key value" pair per line. */
#include <stdio.h>
#include <stdlib.h>

#include "sta.h"

int main(void) {
  const int32_t window[6] = {3, 3, 3, 1, 1, 1};
  sta_problem p = {0};
  p.batch = 1, p.heads = 2, p.head_dim = 128;
  p.T = 12, p.H = 16, p.W = 16;
  p.tile_t = 6, p.tile_h = 8, p.tile_w = 8;
  p.window = window;
  p.scale = 0.f;
  p.flags = STA_PROBLEM_HOST_ONLY | STA_PROBLEM_BACKWARD;
  sta_plan_t plan = NULL;
  sta_status st = sta_plan_create(&p, &plan);
  printf("create %d\n", (int)st);
  if (st != STA_OK) return 1;

  int32_t n_tiles = 0, tau = 0, fwd = 0, bwd = 0;
  sta_plan_geometry(plan, &n_tiles, &tau);
  sta_plan_launches(plan, &fwd, &bwd);
  size_t fwd_bytes = 0, bwd_bytes = 0, host_bytes = 0;
  sta_plan_workspace_size(plan, &fwd_bytes, &bwd_bytes);
  sta_plan_host_workspace_size(plan, &host_bytes);
  printf("tiles %d\ntau %d\nfwd_launches %d\nbwd_launches %d\n", n_tiles, tau, fwd, bwd);
  printf("fwd_bytes %zu\nbwd_bytes %zu\nhost_bytes %zu\n", fwd_bytes, bwd_bytes, host_bytes);

  size_t n = 0;
  sta_plan_kv_tiles(plan, 0, NULL, 0, &n); /* size query */
  int32_t *list = (int32_t *)malloc(n * sizeof(int32_t));
  sta_plan_kv_tiles(plan, 0, list, n, &n);
  printf("kv_entries_head0 %zu\nkv_tile0_first %d\nkv_tile0_last %d\n", n, list[0], list[n / (size_t)n_tiles - 1]);
  free(list);

  /* a compute call on a host-only plan is refused before any launch */
  printf("forward_on_host_plan %d\n", (int)sta_forward(plan, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL, 0));
  sta_plan_destroy(plan);

  p.T = 13; /* the tile no longer divides the latent */
  printf("bad_shape %d\n", (int)sta_plan_create(&p, &plan));
  p.T = 12, p.head_dim = 96;
  printf("bad_head_dim %d\n", (int)sta_plan_create(&p, &plan));
  printf("status_8 %s\n", sta_status_string(STA_ERR_TIMEOUT));
  return 0;
}
