/* A plain C99 caller of the library's host-only entry points, built and run
 * by tests/test_abi_cpu.py without a GPU: the tile plan of the Qwen3-8B QKV
 * projection at 448 rows, the tcgen05 attention's work split for three
 * requests, and a refused plan. One "name value" pair per line, compared
 * there with what the Python binding gets from the same calls. */
#include <stdio.h>

#include "isd.h"

int main(void) {
  int32_t plan[ISD_GEMM_PLAN_FIELDS];
  const int32_t kend[3] = {100, 1500, 4096};
  int32_t segs[64 * ISD_ATTN_SEG_FIELDS];
  int32_t n_segments = 0, max_parts = 0;
  int i, rc;

  rc = isd_gemm_plan(448, 6144, 4096, 0, 8, 148, plan);
  printf("plan_rc %d\n", rc);
  for (i = 0; i < ISD_GEMM_PLAN_FIELDS; ++i) printf("plan %d\n", (int)plan[i]);

  rc = isd_attention_split(3, 7, 32, 8, 128, 64, 64, kend, 16, segs, 64, &n_segments, &max_parts);
  printf("split_rc %d\nsegments %d\nmax_parts %d\n", rc, (int)n_segments, (int)max_parts);
  for (i = 0; i < n_segments * ISD_ATTN_SEG_FIELDS && i < 64 * ISD_ATTN_SEG_FIELDS; ++i)
    printf("seg %d\n", (int)segs[i]);

  rc = isd_gemm_plan(448, 100, 4096, 0, 8, 148, plan);
  printf("refused_rc %d\n", rc);
  return 0;
}
