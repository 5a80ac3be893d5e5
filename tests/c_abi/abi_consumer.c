/* A plain C99 consumer of include/cowa.h: it includes the header as C, links libcowa.so and
 * calls the host-side entry points (no GPU is touched: the compute entry points are only
 * given arguments that fail validation, which happens before any launch).  Prints one
 * "key value..." line per result for the Python test to compare. */
#include <stdio.h>
#include <stdlib.h>

#include "cowa.h"

static cowa_tensor tensor(void* p, int64_t sb, int64_t st, int64_t sh) {
  cowa_tensor t;
  t.ptr = p; t.stride_b = sb; t.stride_t = st; t.stride_h = sh;
  return t;
}

int main(void) {
  cowa_pattern pat = {4, 6, 64, 4, 0, 0, 0.0f};
  int64_t counts[4 * 70];
  int32_t plan[4 * 4096];
  size_t n = 0;
  int g, t, s;
  /* never dereferenced: validation rejects the calls before any launch */
  void* fake = (void*)(uintptr_t)0x10000;
  void* odd = (void*)(uintptr_t)0x10008;
  cowa_tensor q = tensor(fake, 70 * 8 * 64, 8 * 64, 64);
  cowa_tensor kv = tensor(fake, 70 * 4 * 64, 4 * 64, 64);
  float* lse = (float*)fake;

  printf("version %d\n", cowa_version());
  for (s = 0; s <= 6; ++s) printf("status %d %s\n", s, cowa_status_string((cowa_status)s));

  if (cowa_visible_counts(&pat, 4, 70, counts) != COWA_OK) return 1;
  for (g = 0; g < 4; ++g) {
    printf("counts %d", g);
    for (t = 0; t < 70; ++t) printf(" %lld", (long long)counts[g * 70 + t]);
    printf("\n");
  }
  for (s = 0; s < 2; ++s) {
    size_t i;
    if (cowa_plan_debug(&pat, 4, 70, 32, 16, s, plan, 4096, &n, NULL) != COWA_OK) return 2 + s;
    for (i = 0; i < n; ++i)
      printf("%s %d %d %d %d\n", s == 0 ? "fwd_plan" : "bwd_plan", plan[4 * i], plan[4 * i + 1], plan[4 * i + 2],
             plan[4 * i + 3]);
  }

  {
    cowa_pattern big = {128, 4096, 131072, 8, 0, 0, 0.0f};
    printf("compact_rows %d\n", cowa_compact_rows(&big, 8));
  }
  printf("fwd_workspace %zu\n", cowa_fwd_workspace_size(&pat, 1, 70, 8, 4, 64));
  /* argument errors, each returned before any launch */
  printf("err_null_pattern %d\n", (int)cowa_fwd(NULL, 1, 70, 8, 4, 64, q, kv, kv, q, lse, fake, 256, NULL));
  printf("err_head_dim %d\n", (int)cowa_fwd(&pat, 1, 70, 8, 4, 96, q, kv, kv, q, lse, fake, 256, NULL));
  printf("err_group %d\n", (int)cowa_fwd(&pat, 1, 70, 8, 3, 64, q, kv, kv, q, lse, fake, 256, NULL));
  printf("err_align %d\n", (int)cowa_fwd(&pat, 1, 70, 8, 4, 64, tensor(odd, 70 * 8 * 64, 8 * 64, 64), kv, kv, q,
                                         lse, fake, 256, NULL));
  printf("err_workspace %d\n", (int)cowa_fwd(&pat, 1, 70, 8, 4, 64, q, kv, kv, q, lse, fake, 0, NULL));
  {
    cowa_pattern bad = pat;
    bad.D = 3; /* does not divide H = 4 */
    printf("err_pattern %d\n", (int)cowa_fwd(&bad, 1, 70, 8, 4, 64, q, kv, kv, q, lse, fake, 256, NULL));
    bad = pat;
    bad.kv_head_base = 2; bad.h_kv_global = 4; /* heads 2..5 of a 4-head layer */
    printf("err_tp_range %d\n", (int)cowa_fwd(&bad, 1, 70, 8, 4, 64, q, kv, kv, q, lse, fake, 256, NULL));
  }
  return 0;
}
