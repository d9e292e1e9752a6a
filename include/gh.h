/*
 * gh.h — C ABI of libgh, next-token cross-entropy for NVIDIA B200 (sm_100a).
 *
 * Operations from the Greyhound functional API (greyhound.nn.functional):
 *
 *  - gh_ce_fwd_bwd: `cross_entropy` — materialised [B, V] logits and [B]
 *    targets; the summed (or mean) loss with optional z-loss and the logits
 *    gradient, both from the same call (one read of each row from HBM).  nuvec
 *    FastOp::CrossEntropy gives the row loss logsumexp(x) - x[target]
 *    (float32) and FastOp::CrossEntropyVjp its logits gradient.
 *  - gh_ce_fwd: the same loss without the gradient (evaluation; Gpt2 `loss`,
 *    viv `gpt_loss`), optionally unreduced.
 *  - gh_selective_log_softmax: `selective_log_softmax` — one log-probability
 *    per row, x[index] - logsumexp(x), without the full log-softmax.
 *  - gh_ce_vjp: nuvec `FastOp::CrossEntropyVjp` — the logits gradient for a
 *    per-row upstream gradient, from the forward's row loss.
 *  - gh_chunked_linear_loss: `chunked_linear_loss` — the chunk loop of
 *    gh_linear_ce with a caller-provided loss and logits gradient per chunk.
 *  - gh_linear_ce: `chunked_linear_cross_entropy` — logits = inputs @ weight.T
 *    computed one row chunk at a time and never materialised in full; per
 *    chunk the logits gradient G gives grad_inputs[chunk] = G @ weight and
 *    grad_weight += G.T @ inputs[chunk] (`chunked_linear_loss`), with the
 *    weight-gradient accumulator in fp32 or in the weight dtype
 *    (`grad_weight_accum_dtype`).
 *
 * Definitions (x = one logits row, t its target, ii = ignore_index,
 * z = z-loss multiplier, lse = log sum_j exp(x_j)):
 *     row loss  = (lse - x_t) + z * lse^2          if t != ii, else 0
 *     grad_j    = scale * ((1 + 2 z lse) * exp(x_j - lse) - [j == t])
 *     scale     = 1 / max(n_valid, 1) for GH_REDUCTION_MEAN, 1 for SUM
 *     loss      = sum of row losses * (1 / max(n_valid, 1) for MEAN)
 * where n_valid counts the targets that are not ii (over the whole call; in
 * linear-CE over all N rows, not per chunk).  Rows whose target equals ii
 * contribute no loss and an all-zero gradient row.  Gradients are those of the
 * returned loss (upstream gradient 1).
 *
 * Common rules for every entry point:
 *  - Tensor pointers are DEVICE pointers owned by the caller, row-major and
 *    contiguous (row stride = number of columns).  The library keeps no
 *    pointer after the call returns.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Work is enqueued on it and the call returns without waiting;
 *    outputs are valid once the stream reaches that point.  The library
 *    allocates its scratch stream-ordered on the same stream, from a memory
 *    pool it keeps per device (freed memory is kept for later calls).
 *  - Arguments are validated on the host before anything is enqueued:
 *    null pointers, negative sizes, unknown enums and non-finite z give
 *    GH_ERR_INVALID_ARG and nothing runs.  B == 0 (or N == 0) writes loss = 0.
 *  - A target outside [0, V) that is not ii violates the precondition; it
 *    cannot be seen on the host without a sync, so the kernels treat that row
 *    as ignored (no out-of-bounds access) and record GH_ERR_TARGET_RANGE in
 *    the device status word (read it with gh_get_device_status).
 *  - Every device-side wait is bounded; a wait that runs out records
 *    GH_ERR_TIMEOUT in the status word and the kernel returns.
 *  - The library is not thread-safe across concurrent calls that share a
 *    stream only in the sense CUDA streams are; distinct streams are fine.
 */
#ifndef GH_H_
#define GH_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GH_OK = 0,
  GH_ERR_INVALID_ARG = 1,  /* rejected on the host; nothing was enqueued */
  GH_ERR_UNSUPPORTED = 2,  /* valid request outside what this library version supports */
  GH_ERR_ALLOC = 3,        /* scratch allocation failed; nothing was enqueued */
  GH_ERR_CUDA = 4,         /* a CUDA runtime/driver call or launch failed */
  GH_ERR_TIMEOUT = 5,      /* a bounded device wait ran out (device status) */
  GH_ERR_TARGET_RANGE = 6  /* a target outside [0, V) was seen (device status) */
} gh_status_t;

/* Greyhound `reduction`: "mean" divides the summed loss by the number of
 * valid tokens, "sum" returns the summed loss. */
typedef enum { GH_REDUCTION_MEAN = 0, GH_REDUCTION_SUM = 1 } gh_reduction_t;

/* Greyhound `grad_weight_accum_dtype`: "fp32" accumulates the per-chunk
 * weight-gradient products in fp32 and casts once at the end; "weight"
 * accumulates in the weight dtype, rounding between chunks. */
typedef enum { GH_ACCUM_FP32 = 0, GH_ACCUM_WEIGHT = 1 } gh_accum_t;

/* Element type of logits / gradients. */
typedef enum { GH_F32 = 0, GH_BF16 = 1 } gh_dtype_t;

/*
 * gh_ce_fwd_bwd — standalone cross-entropy, forward and backward in one call
 * (Greyhound `cross_entropy`).
 *
 *   logits   [B, V] of `dtype` (GH_F32 or GH_BF16), device.
 *   targets  [B] int64 class ids, device.
 *   B >= 0, V >= 1 (V < 2^31).
 *   ignore_index  target value that is ignored (may lie inside [0, V)).
 *   reduction     GH_REDUCTION_MEAN or GH_REDUCTION_SUM.
 *   z_mult        z-loss multiplier (finite; 0 disables).
 *   loss     device float32 scalar, written.
 *   grad     [B, V] of `dtype`, device, written with the logits gradient
 *            (round to nearest even).  grad == logits is allowed (in place,
 *            as the raw kernel helper on the Greyhound page does); any other
 *            overlap is not.
 *   stream   cudaStream_t as void*.
 * Non-finite logits follow the definition: a NaN in a valid row makes the loss
 * NaN and every gradient element of that row NaN; ignored rows are not read.
 */
gh_status_t gh_ce_fwd_bwd(const void* logits, const int64_t* targets, int64_t B, int64_t V,
                          gh_dtype_t dtype, int64_t ignore_index, gh_reduction_t reduction,
                          float z_mult, float* loss, void* grad, void* stream);

/*
 * gh_ce_fwd_bwd_noalloc — gh_ce_fwd_bwd for callers that cannot allocate.
 * The Greyhound API has no counterpart; this entry point exists for callers
 * whose device memory is already owned in full by another allocator (a
 * framework's caching allocator, or a fixed arena planned ahead of time),
 * where the stream-ordered allocation gh_ce_fwd_bwd makes for its scratch
 * could fail in the middle of a step, and for loops that forbid allocator
 * calls inside a step.
 *
 * Arguments, results and errors are those of gh_ce_fwd_bwd, except:
 *  - B is limited to 65536 rows: the scratch is a fixed array of
 *    256 + 4 * 65536 bytes inside the library's device image, which every GPU
 *    that loads the library keeps until the process exits.  Larger B returns
 *    GH_ERR_UNSUPPORTED and enqueues nothing.
 *  - The call makes no cudaMalloc/cudaFree and no allocating library call.
 *  - The first call with a given device current looks up the array's device
 *    address (cudaGetSymbolAddress) and caches it; make that first call
 *    before any stream capture on that device.
 *  - All calls share the one array and it keeps the last call's contents (the
 *    call clears what must start at zero).  Calls whose GPU work overlaps
 *    (different streams or host threads) race on it; serialise them.
 */
gh_status_t gh_ce_fwd_bwd_noalloc(const void* logits, const int64_t* targets, int64_t B, int64_t V,
                                  gh_dtype_t dtype, int64_t ignore_index, gh_reduction_t reduction,
                                  float z_mult, float* loss, void* grad, void* stream);

/*
 * Data-parallel shards.  A batch split over ranks has one mean: every shard
 * divides by the valid count of the whole batch.  gh_count_valid writes a
 * shard's count; the caller sums the counts over the ranks (one all-reduce of
 * an int64) and passes the total to the _shard entry points, which are
 * gh_ce_fwd_bwd / gh_linear_ce with that count in place of their own.  Their
 * losses and gradients are then the shard's terms of the batch's: the loss is
 * all-reduced (sum), grad_weight too; logits and input gradients are final.
 *
 * gh_count_valid: count = #{targets != ignore_index} over targets[0..N)
 * (int64 device scalar, written); targets outside [0, V) that are not
 * ignore_index record GH_ERR_TARGET_RANGE and are not counted.
 * n_valid_total: device int64 scalar, read by the kernels (8-byte aligned).
 */
gh_status_t gh_count_valid(const int64_t* targets, int64_t N, int64_t V, int64_t ignore_index, int64_t* count,
                           void* stream);
gh_status_t gh_ce_fwd_bwd_shard(const void* logits, const int64_t* targets, int64_t B, int64_t V,
                                gh_dtype_t dtype, int64_t ignore_index, gh_reduction_t reduction, float z_mult,
                                const int64_t* n_valid_total, float* loss, void* grad, void* stream);
gh_status_t gh_linear_ce_shard(const void* inputs, const void* weight, const int64_t* targets, int64_t N,
                               int64_t D, int64_t V, int64_t chunk, gh_accum_t accum_dtype, int64_t ignore_index,
                               gh_reduction_t reduction, float z_mult, const int64_t* n_valid_total, float* loss,
                               void* grad_inputs, void* grad_weight, void* stream);

/*
 * gh_linear_ce_shard_f32 — gh_linear_ce_shard with fp32 accumulation
 * (Greyhound `grad_weight_accum_dtype` "fp32": accumulate in fp32, cast once)
 * whose weight gradient is returned unrounded, so that a data-parallel caller
 * can sum the shards' fp32 accumulators (all-reduce in fp32) and round the
 * batch's sum once, with gh_cast_f32_to_bf16.
 *   grad_weight_f32  [V, D] float32, device, 16-byte aligned, written (not
 *                    added to) with this shard's sum over its chunks of
 *                    G_c^T @ inputs[chunk], in fp32.
 * Other arguments as for gh_linear_ce_shard (no accum_dtype argument).
 *
 * gh_cast_f32_to_bf16 — dst[i] = bf16(src[i]) (round to nearest even) for
 * n elements; src 16-byte aligned, dst 8-byte aligned, device.
 */
gh_status_t gh_linear_ce_shard_f32(const void* inputs, const void* weight, const int64_t* targets, int64_t N,
                                   int64_t D, int64_t V, int64_t chunk, int64_t ignore_index,
                                   gh_reduction_t reduction, float z_mult, const int64_t* n_valid_total,
                                   float* loss, void* grad_inputs, float* grad_weight_f32, void* stream);
gh_status_t gh_cast_f32_to_bf16(const float* src, void* dst, int64_t n, void* stream);

/*
 * gh_linear_ce_shard_f32_sliced — gh_linear_ce_shard_f32 whose last weight-
 * gradient contraction (the last chunk's G^T @ inputs) runs as `dw_slices`
 * launches over consecutive ranges of weight rows, so that a data-parallel
 * caller can start the cross-rank sum of the finished rows while the rest are
 * computed (the weight-gradient reduction overlapped with the chunk loop; the
 * Greyhound functional API's chunked_linear_cross_entropy with fp32
 * grad_weight_accum_dtype, sharded by rows).  The pages have no counterpart for
 * the callback: it is this library's interface for the overlap.
 *
 * After enqueuing the launch for weight rows [v0, v1) the call invokes
 *     on_slice(ctx, v0, v1, stream)
 * on the calling host thread; rows v0 .. v1-1 of grad_weight_f32 are final
 * once the work enqueued on `stream` so far has completed (enqueue the
 * reduction behind it, e.g. an all-reduce ordered after `stream`).  The
 * ranges come in order, cover [0, V) without overlap and start at multiples of
 * 128 (whole output tiles).  on_slice returning anything but GH_OK stops the call, which returns
 * that status.  With N = 0 the only callback is (0, V), after grad_weight_f32
 * is zeroed.
 *   dw_slices  >= 1: the number of ranges (at most one per output tile of
 *              weight rows).
 *   max_sms    the sliced launches use at most this many SMs (<= 0: all), so
 *              that the caller's communication kernels find free SMs.
 * Results are bit-identical to gh_linear_ce_shard_f32 for any dw_slices and
 * max_sms (each output tile is computed by one CTA pair in the same order).
 * Other arguments as for gh_linear_ce_shard_f32.  GH_ERR_INVALID_ARG for
 * dw_slices < 1 or a null on_slice.
 */
typedef gh_status_t (*gh_dw_slice_fn)(void* ctx, int64_t v0, int64_t v1, void* stream);
gh_status_t gh_linear_ce_shard_f32_sliced(const void* inputs, const void* weight, const int64_t* targets,
                                          int64_t N, int64_t D, int64_t V, int64_t chunk, int64_t ignore_index,
                                          gh_reduction_t reduction, float z_mult, const int64_t* n_valid_total,
                                          float* loss, void* grad_inputs, float* grad_weight_f32, int64_t dw_slices,
                                          int max_sms, gh_dw_slice_fn on_slice, void* ctx, void* stream);

/*
 * gh_ce_fwd — the cross-entropy loss of gh_ce_fwd_bwd without its gradient:
 * the evaluation form (forward only, nothing kept for a backward), reading the
 * logits once.
 *
 *   logits, targets, B, V, dtype, ignore_index, reduction, z_mult, loss
 *            as for gh_ce_fwd_bwd.
 *   row_loss optional device float32 [B] (NULL: not returned); written with
 *            each row's loss before reduction, 0 for ignored rows (the
 *            unreduced loss).
 * Scratch (stream-ordered): 16 bytes, plus 4*B bytes when row_loss is NULL.
 */
gh_status_t gh_ce_fwd(const void* logits, const int64_t* targets, int64_t B, int64_t V,
                      gh_dtype_t dtype, int64_t ignore_index, gh_reduction_t reduction,
                      float z_mult, float* loss, float* row_loss, void* stream);

/*
 * gh_ce_vjp — the logits gradient of the per-row cross-entropy for an upstream
 * gradient per row (nuvec FastOp::CrossEntropyVjp: logits, targets, the
 * forward's row loss and g):
 *     grad_j = g_r (exp(x_j - lse_r) - [j == t_r]),   lse_r = row_loss_r + x_{r,t_r}
 * The forward's row loss carries lse, so the gradient takes one sweep over
 * each row with no reduction.
 *
 *   logits, targets, B, V, dtype, ignore_index  as for gh_ce_fwd_bwd.
 *   row_loss  [B] float32, device: lse - x_t per row without z-loss, as
 *             gh_ce_fwd returns with z_mult = 0 (values of ignored rows are
 *             not read).
 *   g         [B] float32, device: the upstream gradient of each row's loss.
 *   grad      [B, V] of `dtype`, device, written; grad == logits is allowed.
 * Rows whose target equals ignore_index get a zero gradient row; a target
 * outside [0, V) likewise, and records GH_ERR_TARGET_RANGE.  No scratch.
 */
gh_status_t gh_ce_vjp(const void* logits, const int64_t* targets, int64_t B, int64_t V, gh_dtype_t dtype,
                      int64_t ignore_index, const float* row_loss, const float* g, void* grad, void* stream);

/*
 * gh_selective_log_softmax — Greyhound `selective_log_softmax`: for each row
 * r, out[r] = x[r, index[r]] - logsumexp(x[r, :]), the log-probability of one
 * selected class, without materialising the log-probabilities.
 *
 *   logits   [rows, V] of `dtype` (GH_F32 or GH_BF16), device (any leading
 *            shape flattened to rows).
 *   index    [rows] int64, device.
 *   rows >= 0, V >= 1 (V < 2^31).
 *   out      [rows] float32, device, written.
 * No ignore_index: every row is computed.  An index outside [0, V) violates
 * the precondition: that row's logits are not read, out[r] = NaN, and
 * GH_ERR_TARGET_RANGE is recorded in the device status word.  No scratch.
 */
gh_status_t gh_selective_log_softmax(const void* logits, const int64_t* index, int64_t rows, int64_t V,
                                     gh_dtype_t dtype, float* out, void* stream);

/*
 * gh_linear_ce — chunked fused linear cross-entropy (Greyhound
 * `chunked_linear_cross_entropy` over `chunked_linear_loss`).
 *
 *   inputs       [N, D] bf16, device (hidden states, one row per token).
 *   weight       [V, D] bf16, device (LM head; logits = inputs @ weight.T).
 *   targets      [N] int64, device.
 *   N >= 0, D >= 1, V >= 1; D must be a multiple of 8 (16-byte rows for TMA).
 *   chunk        rows per logits chunk; <= 0 selects the default (the largest
 *                multiple of 128 whose bf16 chunk logits fit 1 GiB, capped at N).
 *   accum_dtype  GH_ACCUM_FP32 or GH_ACCUM_WEIGHT.
 *   ignore_index, reduction, z_mult  as for gh_ce_fwd_bwd.
 *   loss         device float32 scalar, written.
 *   grad_inputs  [N, D] bf16, device, written.
 *   grad_weight  [V, D] bf16, device, written (overwritten, not added to).
 *   stream       cudaStream_t as void*.
 * Scratch (stream-ordered): the chunk's exponentials, chunk x round_up(V, 64)
 * bf16 (twice that with fp32 accumulation over several chunks when
 * 2 x chunk x D x 2 bytes <= 32 MiB: two chunks then share one weight-gradient
 * contraction), an fp32 [V, D] accumulator when fp32 accumulation needs more
 * than one contraction, the chunk's scaled inputs (chunk or 2 x chunk rows
 * x D bf16), per-tile row statistics (ceil(V / 256) x chunk float2) and O(N)
 * floats.
 */
gh_status_t gh_linear_ce(const void* inputs, const void* weight, const int64_t* targets,
                         int64_t N, int64_t D, int64_t V, int64_t chunk, gh_accum_t accum_dtype,
                         int64_t ignore_index, gh_reduction_t reduction, float z_mult,
                         float* loss, void* grad_inputs, void* grad_weight, void* stream);

/*
 * gh_chunked_linear_loss — Greyhound `chunked_linear_loss`: the chunked
 * linear projection of gh_linear_ce with a caller-provided loss in place of
 * the cross-entropy.  For each chunk of rows [row0, row0 + rows) the library
 * computes logits = inputs[chunk] @ weight.T into a bf16 buffer and calls
 * `loss_fn` on the calling host thread; `loss_fn` must enqueue on `stream`
 * (it may not wait for it) the work that
 *   - overwrites the logits in place with the logits gradient (bf16, same
 *     layout: row r at logits + r * ld elements, V valid columns), and
 *   - adds the chunk's scalar loss to the float32 device scalar `loss_accum`,
 * and return GH_OK.  The library then forms grad_inputs[chunk] = G @ weight and
 * accumulates grad_weight (+)= G^T @ inputs[chunk] as gh_linear_ce does.
 * The returned loss is the sum of the chunks' losses.  Slicing the caller's
 * per-row arguments to [row0, row0 + rows) is up to `loss_fn` (`ctx`).
 *
 *   inputs, weight, N, D, V, chunk, accum_dtype, grad_inputs, grad_weight,
 *   stream   as for gh_linear_ce.
 *   loss_fn  the callback; ctx is passed through unchanged.
 *   loss     device float32 scalar, written (0 before the first chunk).
 * A status other than GH_OK from loss_fn stops the chunk loop; the library
 * frees its scratch (stream-ordered) and returns that status.
 */
typedef gh_status_t (*gh_chunk_loss_fn)(void* ctx, int64_t row0, int64_t rows, void* logits, int64_t ld,
                                        int64_t V, float* loss_accum, void* stream);

gh_status_t gh_chunked_linear_loss(const void* inputs, const void* weight, int64_t N, int64_t D, int64_t V,
                                   int64_t chunk, gh_accum_t accum_dtype, gh_chunk_loss_fn loss_fn, void* ctx,
                                   float* loss, void* grad_inputs, void* grad_weight, void* stream);

/*
 * gh_get_device_status — synchronises `stream`, returns the first error any
 * kernel recorded on the current device since the last call (GH_OK if none:
 * GH_ERR_TARGET_RANGE or GH_ERR_TIMEOUT), and clears it.  Returns GH_ERR_CUDA
 * if the synchronisation itself fails.
 */
gh_status_t gh_get_device_status(void* stream);

/*
 * Kernel timing (for benchmarks and roofline reports).  Kernel kinds: */
typedef enum {
  GH_KERNEL_CE_ROW = 0,        /* standalone CE row kernel (one per gh_ce_fwd_bwd, gh_ce_fwd,
                                  gh_selective_log_softmax) */
  GH_KERNEL_LOGITS_GEMM = 1,   /* linear-CE: chunk logits = X_c @ W^T (+ CE epilogue) */
  GH_KERNEL_CHUNK_CE = 2,      /* linear-CE: per-chunk loss and logits gradient */
  GH_KERNEL_DX_GEMM = 3,       /* linear-CE: grad_inputs[chunk] = G_c @ W */
  GH_KERNEL_DW_GEMM = 4,       /* linear-CE: grad_weight (+)= G_c^T @ X_c */
  GH_KERNEL_CE_VJP = 5,        /* gh_ce_vjp */
  GH_KERNEL_KINDS = 6
} gh_kernel_t;

/* gh_profile_enable(1) discards earlier records and starts recording a pair
 * of CUDA events around every launch of the kernels above, on the launching
 * stream; gh_profile_enable(0) stops recording (records are kept). */
gh_status_t gh_profile_enable(int enable);

/* Waits for the recorded events of `kind` and returns their summed elapsed
 * milliseconds and the number of launches recorded.  Either output may be
 * NULL.  Returns GH_ERR_INVALID_ARG for an unknown kind, GH_ERR_CUDA if an
 * event query fails. */
gh_status_t gh_profile_read(gh_kernel_t kind, double* total_ms, int64_t* launches);

/* Number of kernels this library has launched in this process (all kinds,
 * including the small counting/reduction kernels). */
int64_t gh_launch_count(void);

/*
 * gh_debug_set — knobs for testing the library's failure path; the Greyhound
 * API has no counterpart.  Every device-side wait in the library is bounded:
 * when one runs out, the kernel records GH_ERR_TIMEOUT, all its roles stop,
 * copies already in flight are waited for, TMEM is freed and the kernel
 * returns.  These knobs make such a wait run out on purpose, so that path can
 * be exercised without faulting or hanging the GPU:
 *
 *   GH_DEBUG_WAIT_LIMIT_NS       the wait limit of every later launch on the
 *                                current device, in ns (value <= 0: back to the
 *                                default of 2 s).  Synchronous.
 *   GH_DEBUG_WITHHOLD_RING_PIECE the next launch of the two-pass cross-entropy
 *                                ring leaves out the copy of piece `value` of
 *                                its first CTA (-1: none); the launch resets it.
 *   GH_DEBUG_WITHHOLD_GEMM_STAGE the next linear cross-entropy GEMM launch
 *                                leaves out the operand loads of stage `value`
 *                                of its first CTA (pair) (-1: none); the launch
 *                                resets it.
 * Off by default; not for production use.  Returns GH_ERR_INVALID_ARG for an
 * unknown knob, GH_ERR_CUDA if the device copy fails.
 */
typedef enum {
  GH_DEBUG_WAIT_LIMIT_NS = 0,
  GH_DEBUG_WITHHOLD_RING_PIECE = 1,
  GH_DEBUG_WITHHOLD_GEMM_STAGE = 2
} gh_debug_t;
gh_status_t gh_debug_set(gh_debug_t knob, int64_t value);

/*
 * gh_exp2_eval — out[i] = 2^y[i] for i < n by one of the two routes the
 * cross-entropy kernels use for their exponentials, so each can be checked on
 * its own (diagnostic; the Greyhound API has no counterpart):
 *   method 0  ex2.approx.ftz.f32 on the MUFU pipe (every kernel; results below
 *             2^-126 flush to zero);
 *   method 1  the FMA-pipe form of the two-pass ring's long rows: y clamped at
 *             -125, split into r = round(y) and f = y - r in [-0.5, 0.5], 2^f
 *             from a degree-5 polynomial fitted to its relative error on that
 *             interval, r added to the exponent field.  Defined for y <= 0 (the
 *             kernels' arguments are differences from a running maximum).
 * y and out: n float32 values, device, caller-owned; may be the same buffer.
 * Asynchronous on `stream`.  GH_ERR_INVALID_ARG for n < 0, an unknown method
 * or a NULL pointer with n > 0; GH_ERR_UNSUPPORTED for n > 2^32; GH_ERR_CUDA
 * if the launch fails.
 */
gh_status_t gh_exp2_eval(const float* y, float* out, int64_t n, int method, void* stream);

/* Static, NUL-terminated description of a status code. */
const char* gh_status_string(gh_status_t status);

/* Library version string, e.g. "gh 0.1.0 sm_100a". */
const char* gh_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GH_H_ */
