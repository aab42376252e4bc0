/* Calls libmxa.so's host-side entry points from plain C (no GPU needed) and
 * prints one line per check; the Python test compiles and runs it. */
#include <stdio.h>
#include <string.h>

#include "mxa.h"

int main(void) {
  /* long-context decode: B=2, Hq=64, Hkv=8, D=128, pages of 64, 16384 keys */
  mxa_decode_params_t p = {2, 1, 64, 8, 128, 512, 64, 256, 16384, MXA_BF16};
  mxa_plan_t plan;
  memset(&plan, 0, sizeof plan);
  mxa_status_t st = mxa_plan(&p, 0, 148, &plan);
  printf("plan %d schedule %d grid %d units %d unit_cost %d combine %d ws %zu\n", (int)st, plan.schedule,
         plan.grid, plan.units, plan.unit_cost, plan.needs_combine, plan.workspace_bytes);
  st = mxa_plan(&p, 4, 148, &plan);
  printf("uniform %d schedule %d grid %d splits %d\n", (int)st, plan.schedule, plan.grid, plan.num_splits);
  /* the first phase of the two-phase call, from C: the uniform plan's size
   * (a host computation) and a refusal */
  printf("wsize %zu %zu %d\n", mxa_decode_workspace_size(&p, 4), plan.workspace_bytes,
         mxa_decode_workspace_size(&p, -1) == (size_t)-1);
  printf("pack %d %d\n", mxa_should_pack_gqa(0, 1, 4, 64), mxa_should_pack_gqa(0, 128, 1, 64));
  printf("splits %d %d\n", mxa_num_splits_heuristic(16, 148, 296, 128, 128, 0, 1, 8388608.0),
         mxa_num_splits_heuristic(256, 148, 296, 32, 64, 0, 1, 1048576.0));
  p.D = 96;
  printf("unsupported %d\n", (int)mxa_plan(&p, 0, 148, &plan));
  p.D = 128;
  /* a run refused before any launch: no workspace for a split plan */
  mxa_plan(&p, 0, 148, &plan);
  st = mxa_decode_fwd_with_plan((void *)4096, (void *)4096, (void *)4096, (const int32_t *)4096,
                                (const int32_t *)4096, &p, 0.125f, 0, &plan, NULL, 0, (void *)4096, NULL, NULL);
  printf("no workspace %d %s\n", (int)st, mxa_status_string(st));
  return 0;
}
