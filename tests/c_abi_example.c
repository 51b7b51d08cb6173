/* A C (not C++) caller of libgnorm: compiles against include/gnorm.h with a C compiler and
 * uses the host-only entry points, which need no GPU.  Built and run by test_abi_cpu.py. */
#include <stdio.h>
#include <string.h>

#include "gnorm.h"

int main(void) {
  gnorm_plan plan;
  int st = gnorm_plan_query(1, 368640, 128, 1, 148, 0, &plan);
  if (st != GNORM_OK) {
    printf("plan failed: %s\n", gnorm_status_string(st));
    return 1;
  }
  size_t ws = gnorm_bwd_workspace_bytes_for(368640, 128, 1, 148);
  gnorm_tuning t;
  memset(&t, 0, sizeof(t));
  t.stage_bytes = 8192;
  gnorm_set_tuning(&t);
  gnorm_plan small;
  gnorm_plan_query(0, 1 << 20, 128, 1, 148, 0, &small);
  gnorm_set_tuning(NULL);
  /* argument checks that precede any CUDA call */
  int null_status = gnorm_fwd(NULL, NULL, NULL, 1e-6f, NULL, NULL, 4, 128, NULL);
  gnorm_fwd_desc d;
  memset(&d, 0, sizeof(d));
  d.M = 4;
  d.N = 100;
  int shape_status = gnorm_fwd_ex(&d, NULL);
  printf("grid=%d rows=%d stages=%d ws=%zu small_rows=%d null=%d shape=%d %s\n", plan.grid,
         plan.rows_per_stage, plan.stages, ws, small.rows_per_stage, null_status, shape_status,
         gnorm_build_info());
  return 0;
}
