// Internal interface of the standalone cross-entropy kernels (ce.cu).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/gh.h"

namespace gh {

// What the row kernel produces per row.
enum CeMode : int {
  kModeFwdBwd = 0,   // row loss and the logits gradient
  kModeFwd = 1,      // row loss only (no gradient; grad may be null)
  kModeSelect = 2    // row value x[index] - lse (selective log-softmax; NaN for an index outside [0, V))
};

struct CeArgs {
  const void* logits;                 // [B, V] row-major
  void* grad;                         // [B, V] row-major, same dtype
  const int64_t* targets;             // [B]
  int64_t V;
  int64_t ld;                         // row stride in elements (>= V)
  int64_t ignore_index;
  float z;                            // z-loss multiplier
  int mean;                           // 1: divide by n_valid
  const unsigned long long* n_valid;  // written by ce_count_kernel
  float* row_loss;                    // [B] per-row values (losses, or the selected log-probabilities)
  int64_t B;                          // rows (set by ce_launch)
  int slice;                          // elements per CTA (set by ce_launch)
  int cluster;                        // CTAs per row (set by ce_launch)
  int buf_bytes;                      // bytes per slice buffer (set by ce_launch)
  int npieces;                        // bulk copies per slice (set by ce_launch)
  int congruent;                      // (logits - grad) % 16 == 0
  int profile_kind;                   // gh_kernel_t the row kernel is timed as
  int mode;                           // CeMode
  int64_t withhold_plus1;             // failure-path tests: 1 + the piece CTA 0's ring producer leaves out (0: none)
};

struct CePlan {
  bool streaming;  // row too long for the shared-memory path
  int cluster;     // CTAs per row
  int slice;       // elements per CTA
  int buf_bytes;   // one slice buffer (two per CTA)
  int smem_bytes;  // dynamic shared memory per CTA
};

CePlan ce_plan(int64_t V, int elem_bytes);
gh_status_t ce_count_launch(const int64_t* targets, int64_t n, int64_t V, int64_t ii,
                            unsigned long long* count, cudaStream_t stream);
gh_status_t ce_launch(const CeArgs& args, int64_t B, gh_dtype_t dtype, cudaStream_t stream);
// Ring pipelines (ce_ring.cu): one persistent CTA per SM (`grid` CTAs), rows
// round-robin over the CTAs; kModeFwd / kModeSelect stream each row once,
// kModeFwdBwd twice (the second copy from L2) and store the gradient.
int ce_ring_smem_bytes();
gh_status_t ce_ring_launch(const CeArgs& args, int elem_bytes, int grid, cudaStream_t stream);
// 2^y[i] -> out[i] by ex2.approx (method 0) or the ring's FMA-pipe polynomial (method 1).
gh_status_t exp2_eval_launch(const float* y, float* out, int64_t n, int method, cudaStream_t stream);
// Per-row cross-entropy VJP (ce_vjp.cu).
gh_status_t ce_vjp_launch(const void* logits, const int64_t* targets, const float* row_loss, const float* g,
                          void* grad, int64_t B, int64_t V, int64_t ignore_index, gh_dtype_t dtype,
                          cudaStream_t stream);
gh_status_t ce_reduce_launch(const float* row_loss, int64_t B, const unsigned long long* n_valid, int mean,
                             float* loss, cudaStream_t stream);

}  // namespace gh
