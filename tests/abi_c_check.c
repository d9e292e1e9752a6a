/* A plain C99 consumer of libgh: include/gh.h must compile as C (not only as
 * C++), the library must link and load from a C program, and every argument
 * check that the header promises to make on the host must answer before any
 * GPU work -- so this program runs on a machine without a GPU.  Built and run
 * by tests/test_abi_host.py; prints one line and exits 0 when every check
 * holds. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "gh.h"

static int failures = 0;

#define EXPECT(cond)                                               \
  do {                                                             \
    if (!(cond)) {                                                 \
      fprintf(stderr, "abi_c_check.c:%d: %s\n", __LINE__, #cond);  \
      ++failures;                                                  \
    }                                                              \
  } while (0)

#define BAD(call) EXPECT((call) == GH_ERR_INVALID_ARG)

/* Well-aligned, non-null addresses in distinct 4 GiB windows; never
 * dereferenced, because each call below is refused before it would be. */
static void* addr(int k) { return (void*)(uintptr_t)(0x7F0000000000ull + ((uint64_t)k << 32)); }

static gh_status_t never_called_slice(void* ctx, int64_t v0, int64_t v1, void* stream) {
  (void)ctx; (void)v0; (void)v1; (void)stream;
  return GH_OK;
}

int main(void) {
  const char* version = gh_version();
  EXPECT(version != NULL && strncmp(version, "gh ", 3) == 0);
  EXPECT(strcmp(gh_status_string(GH_OK), "ok") == 0);
  EXPECT(strcmp(gh_status_string(GH_ERR_TIMEOUT), "device wait timed out") == 0);
  EXPECT(strcmp(gh_status_string((gh_status_t)99), "unknown status") == 0);
  EXPECT(gh_launch_count() >= 0);

  const void* x = addr(0);
  const int64_t* t = (const int64_t*)addr(1);
  float* loss = (float*)addr(2);
  void* grad = addr(3);
  const int64_t* n_total = (const int64_t*)addr(4);
  const float nan = (float)NAN;

  /* gh_ce_fwd_bwd and its variants */
  BAD(gh_ce_fwd_bwd(x, t, -1, 100, GH_BF16, -100, GH_REDUCTION_MEAN, 0.0f, loss, grad, NULL));
  BAD(gh_ce_fwd_bwd(x, t, 16, 0, GH_BF16, -100, GH_REDUCTION_MEAN, 0.0f, loss, grad, NULL));
  BAD(gh_ce_fwd_bwd(x, t, 16, 100, (gh_dtype_t)7, -100, GH_REDUCTION_MEAN, 0.0f, loss, grad, NULL));
  BAD(gh_ce_fwd_bwd(x, t, 16, 100, GH_BF16, -100, (gh_reduction_t)5, 0.0f, loss, grad, NULL));
  BAD(gh_ce_fwd_bwd(x, t, 16, 100, GH_BF16, -100, GH_REDUCTION_SUM, nan, loss, grad, NULL));
  BAD(gh_ce_fwd_bwd(x, t, 16, 100, GH_BF16, -100, GH_REDUCTION_SUM, 0.0f, NULL, grad, NULL));
  BAD(gh_ce_fwd_bwd(NULL, t, 16, 100, GH_BF16, -100, GH_REDUCTION_SUM, 0.0f, loss, grad, NULL));
  BAD(gh_ce_fwd_bwd_noalloc(x, t, 16, 100, GH_F32, -100, GH_REDUCTION_SUM, 0.0f, loss, NULL, NULL));
  BAD(gh_ce_fwd_bwd_shard(x, t, 16, 100, GH_BF16, -100, GH_REDUCTION_MEAN, 0.0f, NULL, loss, grad, NULL));
  BAD(gh_ce_fwd(x, t, 16, 100, GH_BF16, -100, GH_REDUCTION_MEAN, 0.0f, NULL, NULL, NULL));
  BAD(gh_ce_vjp(x, t, 16, 100, GH_BF16, -100, NULL, (const float*)addr(5), grad, NULL));
  BAD(gh_selective_log_softmax(x, t, -3, 100, GH_BF16, (float*)addr(5), NULL));
  BAD(gh_count_valid(t, -1, 100, -100, (int64_t*)addr(5), NULL));

  /* linear cross-entropy: D must be a multiple of 8, enums known, z finite */
  BAD(gh_linear_ce(x, addr(5), t, 64, 12, 100, 0, GH_ACCUM_FP32, -100, GH_REDUCTION_MEAN, 0.0f, loss, grad,
                   addr(6), NULL));
  BAD(gh_linear_ce(x, addr(5), t, 64, 64, 100, 0, (gh_accum_t)3, -100, GH_REDUCTION_MEAN, 0.0f, loss, grad,
                   addr(6), NULL));
  BAD(gh_linear_ce(x, addr(5), t, 64, 64, 100, 0, GH_ACCUM_WEIGHT, -100, GH_REDUCTION_MEAN, nan, loss, grad,
                   addr(6), NULL));
  BAD(gh_linear_ce_shard(x, addr(5), t, 64, 64, 100, 0, GH_ACCUM_FP32, -100, GH_REDUCTION_MEAN, 0.0f, NULL, loss,
                         grad, addr(6), NULL));
  BAD(gh_linear_ce_shard_f32(x, addr(5), t, 64, 64, 100, 0, -100, GH_REDUCTION_MEAN, 0.0f, n_total, loss, grad,
                             NULL, NULL));
  BAD(gh_linear_ce_shard_f32_sliced(x, addr(5), t, 64, 64, 100, 0, -100, GH_REDUCTION_MEAN, 0.0f, n_total, loss,
                                    grad, (float*)addr(6), 0, 0, never_called_slice, NULL, NULL));
  BAD(gh_linear_ce_shard_f32_sliced(x, addr(5), t, 64, 64, 100, 0, -100, GH_REDUCTION_MEAN, 0.0f, n_total, loss,
                                    grad, (float*)addr(6), 2, 0, NULL, NULL, NULL));
  BAD(gh_chunked_linear_loss(x, addr(5), 64, 64, 100, 0, GH_ACCUM_FP32, NULL, NULL, loss, grad, addr(6), NULL));
  BAD(gh_cast_f32_to_bf16((const float*)addr(5), grad, -1, NULL));

  /* diagnostics */
  BAD(gh_exp2_eval((const float*)addr(5), (float*)addr(6), -1, 0, NULL));
  BAD(gh_exp2_eval((const float*)addr(5), (float*)addr(6), 4, 2, NULL));
  BAD(gh_exp2_eval(NULL, NULL, 4, 1, NULL));
  EXPECT(gh_exp2_eval((const float*)addr(5), (float*)addr(6), ((int64_t)1 << 32) + 1, 0, NULL) == GH_ERR_UNSUPPORTED);
  BAD(gh_profile_read((gh_kernel_t)GH_KERNEL_KINDS, NULL, NULL));
  BAD(gh_debug_set((gh_debug_t)9, 0));
  EXPECT(gh_debug_set(GH_DEBUG_WITHHOLD_RING_PIECE, -1) == GH_OK);

  printf("%s: %d failed checks\n", version, failures);
  return failures != 0;
}
