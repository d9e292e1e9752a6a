// Internal interface of the chunked linear cross-entropy (linear_ce.cu).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/gh.h"

namespace gh {

struct LinearCeArgs {
  const void* X;           // [N, D] bf16
  const void* W;           // [V, D] bf16
  const int64_t* targets;  // [N]
  int64_t N, D, V;
  int64_t chunk;           // <= 0: default
  gh_accum_t accum;
  int64_t ignore_index;
  int mean;
  float z;
  float* loss;             // device scalar
  void* dX;                // [N, D] bf16
  void* dW;                // [V, D] bf16
  gh_chunk_loss_fn loss_fn;  // null: cross-entropy; else the caller's loss per chunk
  void* loss_ctx;
  const unsigned long long* n_total;  // non-null: the mean divides by this count (all shards)
  float* dW32;             // non-null (fp32 accumulation only): grad_weight is returned here as the
                           // unrounded fp32 sum over the chunks, [V, D], and dW is not written
  // dW32 only: the last chunk's weight-gradient launch in dw_slices ranges of
  // weight rows on at most max_sms SMs, on_slice called after each (null: one launch)
  gh_dw_slice_fn on_slice;
  void* slice_ctx;
  int64_t dw_slices;
  int max_sms;
};

// out[i] = bf16(src[i]) (round to nearest even), n elements.
gh_status_t cast_f32_bf16_launch(const float* src, void* out, int64_t n, cudaStream_t stream);

gh_status_t linear_ce_run(const LinearCeArgs& a, cudaStream_t stream);

gh_status_t scratch_alloc(void** p, size_t bytes, cudaStream_t stream);
void scratch_free(void* p, cudaStream_t stream);

}  // namespace gh
