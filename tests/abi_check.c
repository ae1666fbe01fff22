/* A plain C99 caller of libwall: include/wall.h must compile as C, every
 * declared function must resolve at link time, and the host-side argument
 * checks must answer without a GPU (every call below is refused or sized
 * before any CUDA call).  Exits 0 when every check holds, else prints the
 * failing line. */
#include <stdint.h>
#include <stdio.h>

#include "wall.h"

#define CHECK(cond)                                          \
  do {                                                       \
    if (!(cond)) {                                           \
      fprintf(stderr, "abi_check:%d: %s\n", __LINE__, #cond); \
      return 1;                                              \
    }                                                        \
  } while (0)

typedef void (*any_fn)(void);

int main(void) {
  /* an aligned address that is never dereferenced: the calls fail their
     checks first */
  void* const fake = (void*)(uintptr_t)4096;
  float* const ffake = (float*)fake;
  /* every entry point of the header, so the link must resolve each one */
  const any_fn fns[] = {
      (any_fn)wall_version,           (any_fn)wall_error_string,
      (any_fn)wall_prefix_cumsum,     (any_fn)wall_attn_fwd_workspace,
      (any_fn)wall_attn_fwd,          (any_fn)wall_attn_fwd_gate_workspace,
      (any_fn)wall_attn_fwd_gate,     (any_fn)wall_attn_bwd_workspace,
      (any_fn)wall_attn_bwd,          (any_fn)wall_build_kv_cache,
      (any_fn)wall_attn_decode_workspace, (any_fn)wall_attn_decode,
      (any_fn)wall_attn_decode_noalloc,   (any_fn)wall_decode_step_workspace,
      (any_fn)wall_decode_step,       (any_fn)wall_attn_decode_chunk_workspace,
      (any_fn)wall_attn_decode_chunk, (any_fn)wall_get_status,
      (any_fn)wall_selftest_wait_timeout, (any_fn)wall_timing_enable,
      (any_fn)wall_timing_enable_slots,   (any_fn)wall_timing_read,
      (any_fn)wall_attn_bwd_workspace_min,
  };
  for (size_t i = 0; i < sizeof(fns) / sizeof(fns[0]); ++i) CHECK(fns[i] != NULL);

  CHECK(wall_version() >= 1);
  CHECK(wall_error_string(WALL_ERR_INVALID_ARG) != NULL);

  /* HQ % H != 0 */
  CHECK(wall_attn_fwd(fake, fake, fake, ffake, WALL_BF16, 1, 64, 3, 4, 64, 64, 0.f, NULL, NULL,
                      0, NULL, 0, fake, ffake, fake, 1u << 20, NULL) == WALL_ERR_INVALID_ARG);
  /* a head size the library does not build */
  CHECK(wall_attn_fwd(fake, fake, fake, ffake, WALL_BF16, 1, 64, 2, 4, 7, 64, 0.f, NULL, NULL,
                      0, NULL, 0, fake, ffake, fake, 1u << 20, NULL) == WALL_ERR_UNSUPPORTED);
  /* an empty problem is valid and launches nothing */
  CHECK(wall_attn_fwd(fake, fake, fake, ffake, WALL_BF16, 1, 0, 2, 4, 64, 64, 0.f, NULL, NULL,
                      0, NULL, 0, fake, ffake, fake, 0, NULL) == WALL_OK);
  CHECK(wall_attn_fwd_workspace(WALL_BF16, 1, 8192, 4, 16, 128, 128, 0, 0) > 0);
  CHECK(wall_attn_bwd_workspace_min(WALL_BF16, 1, 8192, 4, 16, 128, 128, 0, 0) <
        wall_attn_bwd_workspace(WALL_BF16, 1, 8192, 4, 16, 128, 128, 0, 0, 0));
  CHECK(wall_attn_bwd_workspace(WALL_BF16, 1, 8192, 4, 16, 128, 128, 0, 0, 0) >
        wall_attn_fwd_workspace(WALL_BF16, 1, 8192, 4, 16, 128, 128, 0, 0));
  /* decode: the current token's key must be cached (T_kv >= 1) */
  CHECK(wall_attn_decode(fake, fake, ffake, fake, ffake, NULL, 0.f, 64, WALL_BF16, 1, 0, 10, 2,
                         4, 64, 64, fake, ffake, fake, 1u << 20, NULL) == WALL_ERR_INVALID_ARG);
  CHECK(wall_attn_decode_workspace(32, 32768, 8, 32, 128, 64) > 0);
  /* a slot mask beyond the timed stages */
  CHECK(wall_timing_enable_slots(1u << 31) == WALL_ERR_INVALID_ARG);
  CHECK(wall_timing_enable(0) == WALL_OK);
  printf("abi_check: ok (%d entry points)\n", (int)(sizeof(fns) / sizeof(fns[0])));
  return 0;
}
