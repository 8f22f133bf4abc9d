/*
 * A plain C99 consumer of libfa.so: includes the public headers, links the library and
 * checks, without a GPU, the host-side behaviour include/fa.h promises (status strings,
 * workspace sizes, argument rejection before any launch).  Built and run by
 * tests/test_c_abi.py; prints one line per failed check and exits non-zero on failure.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "fa.h"
#include "fa_debug.h"

static int failures = 0;

#define CHECK(cond)                                               \
  do {                                                            \
    if (!(cond)) {                                                \
      printf("FAILED line %d: %s\n", __LINE__, #cond);            \
      ++failures;                                                 \
    }                                                             \
  } while (0)

/* Fake, 16-byte-aligned device addresses: the library never dereferences them on the
   paths exercised here (every call below is refused before a launch). */
#define A16 ((void*)(uintptr_t)(1u << 20))
#define AT(off) ((void*)((uintptr_t)(1u << 20) + (off)))

static size_t up256(size_t x) { return (x + 255) / 256 * 256; }

int main(void) {
  /* Version and status strings. */
  CHECK(fa_version() == 100);
  CHECK(strcmp(fa_status_string(FA_OK), "ok") == 0);
  for (int s = FA_ERR_INVALID_ARG; s <= FA_ERR_INTERNAL; ++s) {
    const char* m = fa_status_string(s);
    CHECK(m != NULL && strlen(m) > 0 && strcmp(m, "unknown status") != 0);
  }
  CHECK(strcmp(fa_status_string(4242), "unknown status") == 0);

  /* Backward workspace: the call's status word (256-byte slot), fp32 dQ accumulator, D and
   * the log2-scaled LSE, each 256-byte padded. */
  {
    const int B = 2, H = 3, N = 1000, d = 64;
    const size_t rows = (size_t)B * H * N;
    const size_t padded = (size_t)B * H * ((N + 127) / 128 * 128);
    CHECK(fa_bwd_workspace_bytes(B, H, N, d) == 256 + up256(rows * d * 4) + 2 * up256(padded * 4));
    CHECK(fa_bwd_workspace_bytes(0, H, N, d) == 0);
    CHECK(fa_bwd_workspace_bytes(B, H, -1, d) == 0);
  }

  /* Forward: null pointer, bad sizes, bad scale, head dim, alignment. */
  CHECK(fa_fwd(NULL, A16, A16, A16, A16, 1, 1, 128, 64, 0, 0.125f, NULL) == FA_ERR_INVALID_ARG);
  CHECK(fa_fwd(A16, A16, A16, A16, A16, 0, 1, 128, 64, 0, 0.125f, NULL) == FA_ERR_INVALID_ARG);
  CHECK(fa_fwd(A16, A16, A16, A16, A16, 1, 1, -3, 64, 0, 0.125f, NULL) == FA_ERR_INVALID_ARG);
  CHECK(fa_fwd(A16, A16, A16, A16, A16, 1, 1, 128, 64, 0, NAN, NULL) == FA_ERR_INVALID_ARG);
  CHECK(fa_fwd(A16, A16, A16, A16, A16, 1, 1, 128, 64, 0, 0.0f, NULL) == FA_ERR_INVALID_ARG);
  CHECK(fa_fwd(A16, A16, A16, A16, A16, 1, 1, 128, 96, 0, 0.125f, NULL) == FA_ERR_UNSUPPORTED);
  CHECK(fa_fwd(AT(8), A16, A16, A16, A16, 1, 1, 128, 64, 0, 0.125f, NULL) == FA_ERR_MISALIGNED);

  /* Backward: workspace too small or missing, misaligned workspace. */
  {
    const size_t ws = fa_bwd_workspace_bytes(1, 2, 256, 128);
    CHECK(fa_bwd(A16, A16, A16, A16, A16, A16, A16, A16, A16, 1, 2, 256, 128, 1, 0.1f, A16,
                 ws - 1, NULL) == FA_ERR_WORKSPACE);
    CHECK(fa_bwd(A16, A16, A16, A16, A16, A16, A16, A16, A16, 1, 2, 256, 128, 1, 0.1f, NULL,
                 ws, NULL) == FA_ERR_WORKSPACE);
    CHECK(fa_bwd(A16, A16, A16, A16, A16, A16, A16, A16, A16, 1, 2, 256, 128, 1, 0.1f, AT(16),
                 ws, NULL) == FA_ERR_MISALIGNED);
    CHECK(fa_bwd(A16, A16, A16, A16, A16, A16, A16, A16, A16, 1, 2, 256, 80, 1, 0.1f, A16, ws,
                 NULL) == FA_ERR_UNSUPPORTED);
  }

  /* fp32 path: head dim limits. */
  CHECK(fa_fwd_f32(A16, A16, A16, A16, A16, 1, 1, 16, 130, 0, 0.1f, NULL) == FA_ERR_UNSUPPORTED);
  CHECK(fa_fwd_f32(A16, A16, A16, A16, A16, 1, 1, 16, 6, 0, 0.1f, NULL) == FA_ERR_UNSUPPORTED);

  /* Split-KV: causal needs Nq <= Nk; unknown dtype code. */
  {
    const size_t ws = fa_fwd_splitkv_workspace_bytes(1, 4, 200, 100, 128);
    CHECK(fa_fwd_splitkv(A16, A16, A16, A16, A16, 1, 4, 200, 100, 128, 1, 0.1f, FA_DTYPE_BF16,
                         A16, (size_t)1 << 30, NULL) == FA_ERR_INVALID_ARG);
    CHECK(fa_fwd_splitkv(A16, A16, A16, A16, A16, 1, 4, 4, 100, 128, 0, 0.1f, 7, A16,
                         (size_t)1 << 30, NULL) == FA_ERR_UNSUPPORTED);
    (void)ws;
  }

  /* Block-sparse: more than 1024 key tiles is refused; a missing mask is an argument error. */
  CHECK(fa_fwd_block_sparse(A16, A16, A16, A16, A16, 1, 1, 1024 * 128 + 1, 128, 0, 0.1f, A16,
                            A16, (size_t)1 << 30, NULL) == FA_ERR_UNSUPPORTED);
  CHECK(fa_fwd_block_sparse(A16, A16, A16, A16, A16, 1, 1, 256, 128, 0, 0.1f, NULL, A16,
                            (size_t)1 << 30, NULL) == FA_ERR_INVALID_ARG);

  /* FP8 forward: head dim 128 only. */
  CHECK(fa_fwd_fp8(A16, A16, A16, A16, A16, A16, 1, 1, 256, 64, 0, 0.1f, NULL) ==
        FA_ERR_UNSUPPORTED);

  /* A status word must be 4-byte aligned; checked before the device is touched. */
  CHECK(fa_read_device_status(AT(2), NULL) == FA_ERR_MISALIGNED);

  if (failures == 0) printf("c abi: all checks passed\n");
  return failures == 0 ? 0 : 1;
}
