/* Host-side allocation failure in the planner, injected without a GPU: the
 * process caps its own address space (setrlimit RLIMIT_AS) a little above what
 * it uses, then asks for a host-only plan whose KV-tile lists need several GB.
 * The planner must report STA_ERR_OOM, leave *out untouched, and a small plan
 * made afterwards must still succeed.  Prints "key value" lines. */
#include <stdio.h>
#include <stdlib.h>
#include <sys/resource.h>

#include "sta.h"

static long vm_bytes(void) {
  FILE *f = fopen("/proc/self/statm", "r");
  long pages = 0;
  if (!f) return -1;
  if (fscanf(f, "%ld", &pages) != 1) pages = -1;
  fclose(f);
  return pages < 0 ? -1 : pages * 4096L;
}

static sta_status plan_w(int32_t W, int32_t ww, sta_plan_t *out) {
  const int32_t window[3] = {1, 1, ww};
  sta_problem p = {0};
  p.batch = 1, p.heads = 1, p.head_dim = 64;
  p.T = 1, p.H = 1, p.W = W;
  p.tile_t = 1, p.tile_h = 1, p.tile_w = 8;
  p.window = window;
  p.flags = STA_PROBLEM_HOST_ONLY;
  return sta_plan_create(&p, out);
}

int main(void) {
  const long vm = vm_bytes();
  if (vm <= 0) return 2;
  struct rlimit rl;
  rl.rlim_cur = rl.rlim_max = (rlim_t)(vm + (512L << 20));
  if (setrlimit(RLIMIT_AS, &rl) != 0) return 3;

  /* 47104 tiles x 30000 key tiles = 1.41e9 list entries (5.7 GB): inside the
   * 32-bit limit, far above the address space left */
  sta_plan_t big = (sta_plan_t)0x1;
  const sta_status st = plan_w(376832, 30000, &big);
  printf("big_status %d\n", (int)st);
  printf("big_untouched %d\n", big == (sta_plan_t)0x1);

  sta_plan_t small = NULL;
  const sta_status st2 = plan_w(4096, 3, &small);
  printf("small_status %d\n", (int)st2);
  if (st2 == STA_OK) sta_plan_destroy(small);
  return 0;
}
