/*
 * A plain C99 client of libgdattn: only <gdattn.h>, linked against the shared
 * library, no CUDA headers.  Every call below is refused by a host-side check
 * before the library touches CUDA, so it runs on a machine with no GPU; the
 * fake device address is never dereferenced.  Exit status 0 when every call
 * returns the status its header documents, else the number of mismatches.
 */
#include <stdint.h>
#include <stdio.h>

#include "gdattn.h"

static int failures = 0;

static void expect(const char *what, gdattn_status got, gdattn_status want) {
  if (got != want) {
    printf("%s: got %d (%s), want %d (%s)\n", what, (int)got, gdattn_status_string(got),
           (int)want, gdattn_status_string(want));
    ++failures;
  }
}

int main(void) {
  void *const A = (void *)(uintptr_t)0x100000; /* 16-byte aligned, never dereferenced */
  void *const A8 = (void *)(uintptr_t)0x100008;
  float *const F = (float *)A;

  if (gdattn_version() <= 0) {
    printf("gdattn_version: %d\n", (int)gdattn_version());
    ++failures;
  }
  for (int s = 0; s <= 7; ++s)
    if (gdattn_status_string((gdattn_status)s) == NULL) {
      printf("gdattn_status_string(%d) is NULL\n", s);
      ++failures;
    }

  /* a sliding layer: 16 query heads over 8 KV heads, head_dim 256, ring of 1024 */
  gdattn_layer_desc d = {0};
  d.n_q_heads = 16;
  d.n_kv_heads = 8;
  d.head_dim = 256;
  d.window = 1024;
  d.scale = 0.0625f;
  d.cache_capacity = 1024;

  expect("decode, q NULL",
         gdattn_decode(NULL, A, A, A, 1, 8, &d, A, F, A, 1u << 20, NULL),
         GDATTN_ERR_INVALID_ARG);
  expect("decode, q misaligned",
         gdattn_decode(A8, A, A, A, 1, 8, &d, A, F, A, 1u << 20, NULL),
         GDATTN_ERR_MISALIGNED);
  expect("decode, no workspace",
         gdattn_decode(A, A, A, A, 1, 8, &d, A, F, NULL, 0, NULL),
         GDATTN_ERR_WORKSPACE);
  expect("decode, batch 0",
         gdattn_decode(A, A, A, A, 0, 8, &d, A, F, A, 1u << 20, NULL),
         GDATTN_ERR_INVALID_ARG);

  gdattn_layer_desc bad = d;
  bad.n_q_heads = 12; /* not a multiple of the KV heads */
  expect("decode, 12 query heads over 8",
         gdattn_decode(A, A, A, A, 1, 8, &bad, A, F, A, 1u << 20, NULL),
         GDATTN_ERR_INVALID_ARG);
  bad = d;
  bad.head_dim = 128;
  expect("decode, head_dim 128",
         gdattn_decode(A, A, A, A, 1, 8, &bad, A, F, A, 1u << 20, NULL),
         GDATTN_ERR_UNSUPPORTED);

  expect("combine, o_partial NULL",
         gdattn_combine(NULL, F, 1, 16, 2, 256, A, F, NULL), GDATTN_ERR_INVALID_ARG);
  expect("workspace_init, NULL", gdattn_workspace_init(NULL, 1024, NULL),
         GDATTN_ERR_WORKSPACE);
  expect("decode_multi, no tokens",
         gdattn_decode_multi(A, A, A, A, 1, 0, 2048, &d, A, F, A, 1u << 24, NULL),
         GDATTN_ERR_INVALID_ARG);
  expect("decode_fp8, scales NULL",
         gdattn_decode_fp8(A, A, A, NULL, F, A, 1, 8, &d, A, F, A, 1u << 20, NULL),
         GDATTN_ERR_INVALID_ARG);
  if (gdattn_workspace_size(0, 8, &d) != 0) {
    printf("gdattn_workspace_size(batch 0) is not 0\n");
    ++failures;
  }
  return failures;
}
