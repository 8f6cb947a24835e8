/* Compiled as C99 against include/fa.h and linked to libfa.so by tests/test_c_abi.py: the
 * boundary is plain C (no C++ and no torch types), and every argument check answers before
 * any CUDA call, so this runs on a machine without a GPU.  Prints one line per failed check
 * and exits with the number of failures. */
#include <stdio.h>
#include <string.h>

#include "fa.h"

static int failures = 0;
#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      printf("failed: %s (line %d)\n", #cond, __LINE__);              \
      ++failures;                                                     \
    }                                                                 \
  } while (0)

int main(void) {
  void* fake = (void*)(size_t)0x10000;   /* 16-byte aligned, never dereferenced */
  fa_fwd_args fa;
  fa_bwd_args ba;
  fa_fwd_fp8_args f8;
  fa_fwd_partial_args pa;

  CHECK(strcmp(fa_status_string(FA_OK), "FA_OK") == 0);
  CHECK(strcmp(fa_status_string(FA_ERR_RANGE), "FA_ERR_RANGE") == 0);
  CHECK(fa_bwd_workspace_bytes(1, 1, 128, 64) == 128 * 64 * 4 + 2 * 512);
  CHECK(fa_bwd_workspace_bytes_ex(1, 1, 128, 64, 1) == 128 * 64 * 8 + 2 * 512);
  CHECK(fa_bwd_workspace_bytes(1, 1, 128, 96) == 0);
  CHECK(fa_fwd_fp8_workspace_bytes(1, 1, 256, 128) == 128 * 256);
  CHECK(fa_fwd_splitkv_workspace_bytes(1, 1, 128, 64, 2) == 2 * (128 * 64 * 4 + 512));
  CHECK(fa_splitkv_choose(1, 1, 16384, 0, 148) == 2);
  CHECK(fa_splitkv_choose(64, 16, 1024, 0, 148) == 1);

  CHECK(fa_fwd(fake, fake, fake, fake, (float*)fake, 1, 1, 128, 96, 0.125f, 0, NULL, NULL) == FA_ERR_UNSUPPORTED);
  CHECK(fa_fwd(NULL, fake, fake, fake, (float*)fake, 1, 1, 128, 64, 0.125f, 0, NULL, NULL) == FA_ERR_INVALID_ARG);

  memset(&fa, 0, sizeof fa);
  fa.q = fake; fa.k = fake; fa.v = fake; fa.o = fake; fa.lse = (float*)fake;
  fa.B = 1; fa.H = 1; fa.N = 128; fa.d = 64; fa.scale = 0.125f; fa.dtype = FA_BF16;
  fa.dropout_p = 1.0f;                                   /* outside [0, 1) */
  CHECK(fa_fwd_ex(&fa) == FA_ERR_INVALID_ARG);
  fa.dropout_p = 0.0f; fa.dtype = 7;
  CHECK(fa_fwd_ex(&fa) == FA_ERR_UNSUPPORTED);

  memset(&ba, 0, sizeof ba);
  ba.q = ba.k = ba.v = ba.o = ba.dout = fake; ba.lse = (const float*)fake;
  ba.dq = ba.dk = ba.dv = fake;
  ba.B = 1; ba.H = 1; ba.N = 128; ba.d = 64; ba.scale = 0.125f; ba.dtype = FA_BF16;
  ba.workspace = (void*)(size_t)0x100000; ba.deterministic = 1;
  ba.workspace_bytes = fa_bwd_workspace_bytes_ex(1, 1, 128, 64, 1) - 1;
  CHECK(fa_bwd_ex(&ba) == FA_ERR_WORKSPACE);
  ba.workspace_bytes = (size_t)1 << 30; ba.query_splits = 2;   /* splits and the deterministic mode */
  CHECK(fa_bwd_ex(&ba) == FA_ERR_UNSUPPORTED);
  ba.deterministic = 0; ba.query_splits = 65;
  CHECK(fa_bwd_ex(&ba) == FA_ERR_INVALID_ARG);
  CHECK(fa_bwd_workspace_bytes_split(1, 1, 128, 64, 2) == fa_bwd_workspace_bytes(1, 1, 128, 64) + 2 * 128 * 64 * 4);
  CHECK(fa_bwd_splitq_choose(1, 1, 16384, 1, 148) == 3);

  memset(&f8, 0, sizeof f8);
  f8.q = f8.k = f8.v = fake; f8.o = fake; f8.lse = (float*)fake;
  f8.descale_q = f8.descale_k = f8.descale_v = 1.0f;
  f8.B = 1; f8.H = 1; f8.N = 128; f8.d = 64; f8.scale = 0.125f;
  CHECK(fa_fwd_fp8(&f8) == FA_ERR_UNSUPPORTED);         /* d must be 128 */

  memset(&pa, 0, sizeof pa);
  pa.q = pa.k = pa.v = fake; pa.o_part = (float*)fake; pa.lse_part = (float*)fake;
  pa.B = 1; pa.H = 1; pa.N = 512; pa.Nk = 128; pa.d = 64; pa.key_offset = 100; pa.scale = 0.125f;
  CHECK(fa_fwd_partial(&pa) == FA_ERR_INVALID_ARG);      /* offset not a multiple of 128 */

  {
    const float* parts[1] = {(const float*)fake};
    CHECK(fa_lse_merge(parts, parts, 0, fake, (float*)fake, 1, 1, 128, 64, FA_BF16, NULL) == FA_ERR_INVALID_ARG);
  }
  CHECK(fa_selftest_wait_timeout(0, NULL, NULL) == FA_ERR_INVALID_ARG);

  /* fa_bwd_noalloc: fa_bwd's argument errors, before any CUDA call; then its size limit */
  CHECK(fa_bwd_noalloc(NULL, fake, fake, fake, (const float*)fake, fake, fake, fake, fake, 1, 1, 128, 64, 0.125f, 0,
                       NULL, NULL) == FA_ERR_INVALID_ARG);
  CHECK(fa_bwd_noalloc(fake, fake, fake, fake, (const float*)fake, fake, fake, fake, fake, 1, 1, 128, 80, 0.125f, 0,
                       NULL, NULL) == FA_ERR_UNSUPPORTED);
  CHECK(fa_bwd_noalloc(fake, fake, fake, fake, (const float*)fake, fake, fake, fake, fake, 64, 16, 16384, 128,
                       0.125f, 0, NULL, NULL) == FA_ERR_WORKSPACE);

  if (failures == 0) printf("c abi ok\n");
  return failures;
}
