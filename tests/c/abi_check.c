/* A plain C99 consumer of the library: compiles against include/fckl.h (no C++,
 * no CUDA headers), links libfckl, and exercises the host-only entry points and
 * the argument checks.  Prints one line per check; exit status 0 when all hold. */
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "fckl.h"

static int failures = 0;
#define CHECK(cond)                                            \
  do {                                                         \
    if (cond) {                                                \
      printf("ok   %s\n", #cond);                              \
    } else {                                                   \
      printf("FAIL %s\n", #cond);                              \
      ++failures;                                              \
    }                                                          \
  } while (0)

int main(void) {
  fckl_problem p;
  memset(&p, 0, sizeof p);
  p.N = 8192; p.H = 3072; p.V = 128256; p.K = 100; p.T = 1.0f; p.chunk = 0;
  p.teacher = FCKL_TEACHER_LOGITS; p.n_valid_total = 0; p.dw_rows = 0;

  CHECK(fckl_resolved_chunk(&p) == 4096);
  size_t ws = fckl_workspace_bytes(&p);
  CHECK(ws >= (size_t)4096 * 128256 * 2);
  CHECK(fckl_host_workspace_bytes(&p) > ws);
  CHECK(strcmp(fckl_status_string(FCKL_OK), "FCKL_OK") == 0);
  CHECK(strcmp(fckl_status_string(FCKL_ERR_WORKSPACE), "FCKL_ERR_WORKSPACE") == 0);

  /* An explicit chunk bounds the dlogits workspace; dw_rows groups chunks. */
  fckl_problem c = p;
  c.chunk = 1024;
  size_t ws1 = fckl_workspace_bytes(&c);
  CHECK(ws1 >= (size_t)1024 * 128256 * 2 && ws1 < (size_t)1024 * 128256 * 2 + (64u << 20));
  c.dw_rows = 4096;
  CHECK(fckl_workspace_bytes(&c) >= ws1 + (size_t)3 * 1024 * 128256 * 2);

  fckl_problem bad = p;
  bad.T = NAN;
  CHECK(fckl_workspace_bytes(&bad) == 0);
  CHECK(fckl_resolved_chunk(&bad) == -1);
  bad = p;
  bad.K = FCKL_K_MAX + 1;
  CHECK(fckl_workspace_bytes(&bad) == 0);
  bad = p;
  bad.dw_rows = -1;
  CHECK(fckl_workspace_bytes(&bad) == 0);

  /* Host-side rejections happen before any device work. */
  char* f = (char*)(uintptr_t)(1u << 20); /* never dereferenced: every call below is rejected */
  CHECK(fckl_fwd_bwd(&p, NULL, f, (int32_t*)f, (float*)f, NULL, (float*)f, NULL, (float*)f,
                     (float*)f, f, ws, NULL) == FCKL_ERR_INVALID_ARG);
  CHECK(fckl_fwd_bwd(&p, f, f, (int32_t*)f, (float*)f, NULL, (float*)f, NULL, (float*)f,
                     (float*)f, f, ws - 1, NULL) == FCKL_ERR_WORKSPACE);
  CHECK(fckl_fwd(&p, f + 8, f, (int32_t*)f, (float*)f, NULL, (float*)f, NULL, f, ws, NULL) ==
        FCKL_ERR_INVALID_ARG);
  CHECK(fckl_check(NULL, NULL) == FCKL_ERR_INVALID_ARG);

  fckl_profile_begin(0u);
  fckl_kernel_stat st[4];
  CHECK(fckl_profile_end(st, 4) == 0);

  printf("%d failure(s)\n", failures);
  return failures == 0 ? 0 : 1;
}
