// C ABI of libgh (declared in include/gh.h): host-side validation, scratch
// management and dispatch to the kernels.
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "ce.h"
#include "common.cuh"
#include "linear_ce.h"
#include "profile.h"

namespace gh {

// Scratch is stream-ordered, from a memory pool the library creates per
// device.  The pool keeps freed memory (release threshold: 4 GiB) so calls do
// not return memory to the driver and map it again every time.
// GH_FAULT_ALLOC=1 makes every scratch allocation fail (host-side fault
// injection for the error path; nothing is enqueued).
static bool fault_alloc() {
  const char* e = std::getenv("GH_FAULT_ALLOC");
  return e && e[0] == '1';
}

static std::mutex g_pool_mu;
static cudaMemPool_t g_pools[64] = {};

static cudaMemPool_t device_pool(int dev) {
  if (dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> g(g_pool_mu);
  if (!g_pools[dev]) {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) {
      (void)cudaGetLastError();
      return nullptr;
    }
    uint64_t keep = 4ull << 30;
    (void)cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    g_pools[dev] = pool;
  }
  return g_pools[dev];
}

gh_status_t scratch_alloc(void** p, size_t bytes, cudaStream_t stream) {
  *p = nullptr;
  if (fault_alloc()) return GH_ERR_ALLOC;
  if (bytes == 0) bytes = 16;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GH_ERR_CUDA;
  cudaMemPool_t pool = device_pool(dev);
  const cudaError_t e = pool ? cudaMallocFromPoolAsync(p, bytes, pool, stream) : cudaMallocAsync(p, bytes, stream);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    *p = nullptr;
    return GH_ERR_ALLOC;
  }
  return GH_OK;
}

void scratch_free(void* p, cudaStream_t stream) {
  if (p) (void)cudaFreeAsync(p, stream);
}

}  // namespace gh

using namespace gh;

extern "C" {

// gh_ce_fwd_bwd and its data-parallel shard form: n_total (device) is the valid
// count of the whole batch, or null to count this call's targets.
static gh_status_t ce_fwd_bwd_impl(const void* logits, const int64_t* targets, int64_t B, int64_t V,
                                   gh_dtype_t dtype, int64_t ignore_index, gh_reduction_t reduction, float z_mult,
                                   const int64_t* n_total, float* loss, void* grad, void* stream_) {
  if (B < 0 || V < 1 || V >= (int64_t(1) << 31)) return GH_ERR_INVALID_ARG;
  if (dtype != GH_F32 && dtype != GH_BF16) return GH_ERR_INVALID_ARG;
  if (reduction != GH_REDUCTION_MEAN && reduction != GH_REDUCTION_SUM) return GH_ERR_INVALID_ARG;
  if (!std::isfinite(z_mult)) return GH_ERR_INVALID_ARG;
  if (!loss) return GH_ERR_INVALID_ARG;
  if (B > 0 && (!logits || !targets || !grad)) return GH_ERR_INVALID_ARG;
  const int es = dtype == GH_F32 ? 4 : 2;
  if ((reinterpret_cast<uintptr_t>(logits) % es) || (reinterpret_cast<uintptr_t>(grad) % es) ||
      (reinterpret_cast<uintptr_t>(targets) % 8) || (reinterpret_cast<uintptr_t>(loss) % 4))
    return GH_ERR_INVALID_ARG;
  if (grad != logits && B > 0) {
    // Partial overlap of grad and logits is not allowed (exact aliasing is).
    const uintptr_t l0 = reinterpret_cast<uintptr_t>(logits), g0 = reinterpret_cast<uintptr_t>(grad);
    const uintptr_t bytes = static_cast<uintptr_t>(B) * static_cast<uintptr_t>(V) * es;
    if (l0 < g0 + bytes && g0 < l0 + bytes) return GH_ERR_INVALID_ARG;
  }
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (B == 0) return cudaMemsetAsync(loss, 0, sizeof(float), stream) == cudaSuccess ? GH_OK : GH_ERR_CUDA;

  void* scratch = nullptr;
  gh_status_t st = scratch_alloc(&scratch, 16 + static_cast<size_t>(B) * sizeof(float), stream);
  if (st != GH_OK) return st;
  unsigned long long* counter = static_cast<unsigned long long*>(scratch);
  float* row_loss = reinterpret_cast<float*>(static_cast<char*>(scratch) + 16);
  const unsigned long long* n_valid = n_total ? reinterpret_cast<const unsigned long long*>(n_total) : counter;

  const int mean = reduction == GH_REDUCTION_MEAN;
  st = n_total ? GH_OK : ce_count_launch(targets, B, V, ignore_index, counter, stream);
  if (st == GH_OK) {
    CeArgs a{};
    a.logits = logits;
    a.grad = grad;
    a.targets = targets;
    a.V = V;
    a.ld = V;
    a.ignore_index = ignore_index;
    a.z = z_mult;
    a.mean = mean;
    a.n_valid = n_valid;
    a.row_loss = row_loss;
    a.congruent = ((reinterpret_cast<uintptr_t>(logits) ^ reinterpret_cast<uintptr_t>(grad)) & 15) == 0;
    st = ce_launch(a, B, dtype, stream);
  }
  if (st == GH_OK) st = ce_reduce_launch(row_loss, B, n_valid, mean, loss, stream);
  scratch_free(scratch, stream);
  return st;
}

gh_status_t gh_ce_fwd_bwd(const void* logits, const int64_t* targets, int64_t B, int64_t V, gh_dtype_t dtype,
                          int64_t ignore_index, gh_reduction_t reduction, float z_mult, float* loss, void* grad,
                          void* stream) {
  return ce_fwd_bwd_impl(logits, targets, B, V, dtype, ignore_index, reduction, z_mult, nullptr, loss, grad, stream);
}

gh_status_t gh_ce_fwd_bwd_shard(const void* logits, const int64_t* targets, int64_t B, int64_t V, gh_dtype_t dtype,
                                int64_t ignore_index, gh_reduction_t reduction, float z_mult,
                                const int64_t* n_valid_total, float* loss, void* grad, void* stream) {
  if (!n_valid_total || (reinterpret_cast<uintptr_t>(n_valid_total) % 8)) return GH_ERR_INVALID_ARG;
  return ce_fwd_bwd_impl(logits, targets, B, V, dtype, ignore_index, reduction, z_mult, n_valid_total, loss, grad,
                         stream);
}

gh_status_t gh_count_valid(const int64_t* targets, int64_t N, int64_t V, int64_t ignore_index, int64_t* count,
                           void* stream_) {
  if (N < 0 || V < 1 || !count || (reinterpret_cast<uintptr_t>(count) % 8)) return GH_ERR_INVALID_ARG;
  if (N > 0 && (!targets || (reinterpret_cast<uintptr_t>(targets) % 8))) return GH_ERR_INVALID_ARG;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (N == 0) return cudaMemsetAsync(count, 0, sizeof(int64_t), stream) == cudaSuccess ? GH_OK : GH_ERR_CUDA;
  return ce_count_launch(targets, N, V, ignore_index, reinterpret_cast<unsigned long long*>(count), stream);
}

gh_status_t gh_ce_fwd(const void* logits, const int64_t* targets, int64_t B, int64_t V, gh_dtype_t dtype,
                     int64_t ignore_index, gh_reduction_t reduction, float z_mult, float* loss, float* row_loss_out,
                     void* stream_) {
  if (B < 0 || V < 1 || V >= (int64_t(1) << 31)) return GH_ERR_INVALID_ARG;
  if (dtype != GH_F32 && dtype != GH_BF16) return GH_ERR_INVALID_ARG;
  if (reduction != GH_REDUCTION_MEAN && reduction != GH_REDUCTION_SUM) return GH_ERR_INVALID_ARG;
  if (!std::isfinite(z_mult)) return GH_ERR_INVALID_ARG;
  if (!loss) return GH_ERR_INVALID_ARG;
  if (B > 0 && (!logits || !targets)) return GH_ERR_INVALID_ARG;
  const int es = dtype == GH_F32 ? 4 : 2;
  if ((reinterpret_cast<uintptr_t>(logits) % es) || (reinterpret_cast<uintptr_t>(targets) % 8) ||
      (reinterpret_cast<uintptr_t>(loss) % 4) || (reinterpret_cast<uintptr_t>(row_loss_out) % 4))
    return GH_ERR_INVALID_ARG;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (B == 0) return cudaMemsetAsync(loss, 0, sizeof(float), stream) == cudaSuccess ? GH_OK : GH_ERR_CUDA;

  // Scratch: the valid-target count, and the row losses unless the caller
  // takes them.
  void* scratch = nullptr;
  const size_t rows_bytes = row_loss_out ? 0 : static_cast<size_t>(B) * sizeof(float);
  gh_status_t st = scratch_alloc(&scratch, 16 + rows_bytes, stream);
  if (st != GH_OK) return st;
  unsigned long long* n_valid = static_cast<unsigned long long*>(scratch);
  float* row_loss = row_loss_out ? row_loss_out : reinterpret_cast<float*>(static_cast<char*>(scratch) + 16);

  const int mean = reduction == GH_REDUCTION_MEAN;
  st = ce_count_launch(targets, B, V, ignore_index, n_valid, stream);
  if (st == GH_OK) {
    CeArgs a{};
    a.logits = logits;
    a.targets = targets;
    a.V = V;
    a.ld = V;
    a.ignore_index = ignore_index;
    a.z = z_mult;
    a.mean = mean;
    a.row_loss = row_loss;
    a.mode = kModeFwd;
    st = ce_launch(a, B, dtype, stream);
  }
  if (st == GH_OK) st = ce_reduce_launch(row_loss, B, n_valid, mean, loss, stream);
  scratch_free(scratch, stream);
  return st;
}

gh_status_t gh_ce_vjp(const void* logits, const int64_t* targets, int64_t B, int64_t V, gh_dtype_t dtype,
                      int64_t ignore_index, const float* row_loss, const float* g, void* grad, void* stream_) {
  if (B < 0 || V < 1 || V >= (int64_t(1) << 31)) return GH_ERR_INVALID_ARG;
  if (dtype != GH_F32 && dtype != GH_BF16) return GH_ERR_INVALID_ARG;
  if (B > 0 && (!logits || !targets || !row_loss || !g || !grad)) return GH_ERR_INVALID_ARG;
  const int es = dtype == GH_F32 ? 4 : 2;
  if ((reinterpret_cast<uintptr_t>(logits) % es) || (reinterpret_cast<uintptr_t>(grad) % es) ||
      (reinterpret_cast<uintptr_t>(targets) % 8) || (reinterpret_cast<uintptr_t>(row_loss) % 4) ||
      (reinterpret_cast<uintptr_t>(g) % 4))
    return GH_ERR_INVALID_ARG;
  if (grad != logits && B > 0) {
    const uintptr_t l0 = reinterpret_cast<uintptr_t>(logits), g0 = reinterpret_cast<uintptr_t>(grad);
    const uintptr_t bytes = static_cast<uintptr_t>(B) * static_cast<uintptr_t>(V) * es;
    if (l0 < g0 + bytes && g0 < l0 + bytes) return GH_ERR_INVALID_ARG;
  }
  if (B == 0) return GH_OK;
  return ce_vjp_launch(logits, targets, row_loss, g, grad, B, V, ignore_index, dtype,
                       static_cast<cudaStream_t>(stream_));
}

gh_status_t gh_selective_log_softmax(const void* logits, const int64_t* index, int64_t rows, int64_t V,
                                     gh_dtype_t dtype, float* out, void* stream_) {
  if (rows < 0 || V < 1 || V >= (int64_t(1) << 31)) return GH_ERR_INVALID_ARG;
  if (dtype != GH_F32 && dtype != GH_BF16) return GH_ERR_INVALID_ARG;
  if (rows > 0 && (!logits || !index || !out)) return GH_ERR_INVALID_ARG;
  const int es = dtype == GH_F32 ? 4 : 2;
  if ((reinterpret_cast<uintptr_t>(logits) % es) || (reinterpret_cast<uintptr_t>(index) % 8) ||
      (reinterpret_cast<uintptr_t>(out) % 4))
    return GH_ERR_INVALID_ARG;
  if (rows == 0) return GH_OK;
  CeArgs a{};
  a.logits = logits;
  a.targets = index;
  a.V = V;
  a.ld = V;
  a.ignore_index = INT64_MIN;  // every in-range index is selected
  a.row_loss = out;
  a.mode = kModeSelect;
  a.profile_kind = GH_KERNEL_CE_ROW;
  return ce_launch(a, rows, dtype, static_cast<cudaStream_t>(stream_));
}

static gh_status_t linear_ce_impl(const void* inputs, const void* weight, const int64_t* targets, int64_t N,
                                  int64_t D, int64_t V, int64_t chunk, gh_accum_t accum_dtype, int64_t ignore_index,
                                  gh_reduction_t reduction, float z_mult, const int64_t* n_total, float* loss,
                                  void* grad_inputs, void* grad_weight, void* stream_, float* grad_weight_f32 = nullptr,
                                  gh_dw_slice_fn on_slice = nullptr, void* slice_ctx = nullptr,
                                  int64_t dw_slices = 1, int max_sms = 0) {
  if (N < 0 || D < 1 || V < 1 || V >= (int64_t(1) << 31) || D >= (int64_t(1) << 31)) return GH_ERR_INVALID_ARG;
  if (D % 8) return GH_ERR_INVALID_ARG;
  if (accum_dtype != GH_ACCUM_FP32 && accum_dtype != GH_ACCUM_WEIGHT) return GH_ERR_INVALID_ARG;
  if (reduction != GH_REDUCTION_MEAN && reduction != GH_REDUCTION_SUM) return GH_ERR_INVALID_ARG;
  if (!std::isfinite(z_mult)) return GH_ERR_INVALID_ARG;
  if (!loss || !weight || !grad_weight) return GH_ERR_INVALID_ARG;
  if (N > 0 && (!inputs || !targets || !grad_inputs)) return GH_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(inputs) % 16) || (reinterpret_cast<uintptr_t>(weight) % 16) ||
      (reinterpret_cast<uintptr_t>(grad_inputs) % 16) || (reinterpret_cast<uintptr_t>(grad_weight) % 16) ||
      (reinterpret_cast<uintptr_t>(targets) % 8) || (reinterpret_cast<uintptr_t>(loss) % 4))
    return GH_ERR_INVALID_ARG;
  LinearCeArgs a{};
  a.X = inputs;
  a.W = weight;
  a.targets = targets;
  a.N = N;
  a.D = D;
  a.V = V;
  a.chunk = chunk;
  a.accum = accum_dtype;
  a.ignore_index = ignore_index;
  a.mean = reduction == GH_REDUCTION_MEAN;
  a.z = z_mult;
  a.loss = loss;
  a.dX = grad_inputs;
  a.dW = grad_weight;
  a.n_total = reinterpret_cast<const unsigned long long*>(n_total);
  a.dW32 = grad_weight_f32;
  a.on_slice = on_slice;
  a.slice_ctx = slice_ctx;
  a.dw_slices = dw_slices;
  a.max_sms = max_sms;
  return linear_ce_run(a, static_cast<cudaStream_t>(stream_));
}

gh_status_t gh_linear_ce(const void* inputs, const void* weight, const int64_t* targets, int64_t N, int64_t D,
                         int64_t V, int64_t chunk, gh_accum_t accum_dtype, int64_t ignore_index,
                         gh_reduction_t reduction, float z_mult, float* loss, void* grad_inputs, void* grad_weight,
                         void* stream) {
  return linear_ce_impl(inputs, weight, targets, N, D, V, chunk, accum_dtype, ignore_index, reduction, z_mult,
                        nullptr, loss, grad_inputs, grad_weight, stream);
}

gh_status_t gh_linear_ce_shard(const void* inputs, const void* weight, const int64_t* targets, int64_t N, int64_t D,
                               int64_t V, int64_t chunk, gh_accum_t accum_dtype, int64_t ignore_index,
                               gh_reduction_t reduction, float z_mult, const int64_t* n_valid_total, float* loss,
                               void* grad_inputs, void* grad_weight, void* stream) {
  if (!n_valid_total || (reinterpret_cast<uintptr_t>(n_valid_total) % 8)) return GH_ERR_INVALID_ARG;
  return linear_ce_impl(inputs, weight, targets, N, D, V, chunk, accum_dtype, ignore_index, reduction, z_mult,
                        n_valid_total, loss, grad_inputs, grad_weight, stream);
}

gh_status_t gh_linear_ce_shard_f32(const void* inputs, const void* weight, const int64_t* targets, int64_t N,
                                   int64_t D, int64_t V, int64_t chunk, int64_t ignore_index,
                                   gh_reduction_t reduction, float z_mult, const int64_t* n_valid_total,
                                   float* loss, void* grad_inputs, float* grad_weight_f32, void* stream) {
  if (!n_valid_total || (reinterpret_cast<uintptr_t>(n_valid_total) % 8)) return GH_ERR_INVALID_ARG;
  if (!grad_weight_f32 || (reinterpret_cast<uintptr_t>(grad_weight_f32) % 16)) return GH_ERR_INVALID_ARG;
  // grad_weight_f32 stands in for the bf16 output in the argument checks
  return linear_ce_impl(inputs, weight, targets, N, D, V, chunk, GH_ACCUM_FP32, ignore_index, reduction, z_mult,
                        n_valid_total, loss, grad_inputs, grad_weight_f32, stream, grad_weight_f32);
}

gh_status_t gh_linear_ce_shard_f32_sliced(const void* inputs, const void* weight, const int64_t* targets,
                                          int64_t N, int64_t D, int64_t V, int64_t chunk, int64_t ignore_index,
                                          gh_reduction_t reduction, float z_mult, const int64_t* n_valid_total,
                                          float* loss, void* grad_inputs, float* grad_weight_f32, int64_t dw_slices,
                                          int max_sms, gh_dw_slice_fn on_slice, void* ctx, void* stream) {
  if (!n_valid_total || (reinterpret_cast<uintptr_t>(n_valid_total) % 8)) return GH_ERR_INVALID_ARG;
  if (!grad_weight_f32 || (reinterpret_cast<uintptr_t>(grad_weight_f32) % 16)) return GH_ERR_INVALID_ARG;
  if (dw_slices < 1 || !on_slice) return GH_ERR_INVALID_ARG;
  return linear_ce_impl(inputs, weight, targets, N, D, V, chunk, GH_ACCUM_FP32, ignore_index, reduction, z_mult,
                        n_valid_total, loss, grad_inputs, grad_weight_f32, stream, grad_weight_f32, on_slice, ctx,
                        dw_slices, max_sms);
}

gh_status_t gh_cast_f32_to_bf16(const float* src, void* dst, int64_t n, void* stream) {
  if (n < 0) return GH_ERR_INVALID_ARG;
  if (n > 0 && (!src || !dst)) return GH_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(src) % 16) || (reinterpret_cast<uintptr_t>(dst) % 8)) return GH_ERR_INVALID_ARG;
  return cast_f32_bf16_launch(src, dst, n, static_cast<cudaStream_t>(stream));
}

gh_status_t gh_exp2_eval(const float* y, float* out, int64_t n, int method, void* stream) {
  if (n < 0 || (method != 0 && method != 1)) return GH_ERR_INVALID_ARG;
  if (n > 0 && (!y || !out)) return GH_ERR_INVALID_ARG;
  if (n > (int64_t(1) << 32)) return GH_ERR_UNSUPPORTED;  // keeps the grid far inside gridDim.x's limit
  return exp2_eval_launch(y, out, n, method, static_cast<cudaStream_t>(stream));
}

gh_status_t gh_chunked_linear_loss(const void* inputs, const void* weight, int64_t N, int64_t D, int64_t V,
                                   int64_t chunk, gh_accum_t accum_dtype, gh_chunk_loss_fn loss_fn, void* ctx,
                                   float* loss, void* grad_inputs, void* grad_weight, void* stream_) {
  if (N < 0 || D < 1 || V < 1 || V >= (int64_t(1) << 31) || D >= (int64_t(1) << 31)) return GH_ERR_INVALID_ARG;
  if (D % 8) return GH_ERR_INVALID_ARG;
  if (accum_dtype != GH_ACCUM_FP32 && accum_dtype != GH_ACCUM_WEIGHT) return GH_ERR_INVALID_ARG;
  if (!loss_fn || !loss || !weight || !grad_weight) return GH_ERR_INVALID_ARG;
  if (N > 0 && (!inputs || !grad_inputs)) return GH_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(inputs) % 16) || (reinterpret_cast<uintptr_t>(weight) % 16) ||
      (reinterpret_cast<uintptr_t>(grad_inputs) % 16) || (reinterpret_cast<uintptr_t>(grad_weight) % 16) ||
      (reinterpret_cast<uintptr_t>(loss) % 4))
    return GH_ERR_INVALID_ARG;
  LinearCeArgs a{};
  a.X = inputs;
  a.W = weight;
  a.N = N;
  a.D = D;
  a.V = V;
  a.chunk = chunk;
  a.accum = accum_dtype;
  a.loss = loss;
  a.dX = grad_inputs;
  a.dW = grad_weight;
  a.loss_fn = loss_fn;
  a.loss_ctx = ctx;
  return linear_ce_run(a, static_cast<cudaStream_t>(stream_));
}

gh_status_t gh_get_device_status(void* stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (cudaStreamSynchronize(stream) != cudaSuccess) return GH_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return GH_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return GH_ERR_CUDA;
  return static_cast<gh_status_t>(v);
}

gh_status_t gh_profile_enable(int enable) {
  ProfileState& s = profile_state();
  std::lock_guard<std::mutex> g(s.mu);
  if (enable) {
    for (auto& r : s.recs) {
      (void)cudaEventSynchronize(r.stop);
      s.pool.push_back(r.start);
      s.pool.push_back(r.stop);
    }
    s.recs.clear();
  }
  s.enabled = enable != 0;
  return GH_OK;
}

gh_status_t gh_profile_read(gh_kernel_t kind, double* total_ms, int64_t* launches) {
  if (kind < 0 || kind >= GH_KERNEL_KINDS) return GH_ERR_INVALID_ARG;
  ProfileState& s = profile_state();
  std::lock_guard<std::mutex> g(s.mu);
  double tot = 0.0;
  int64_t n = 0;
  for (auto& r : s.recs) {
    if (r.kind != kind) continue;
    if (cudaEventSynchronize(r.stop) != cudaSuccess) return GH_ERR_CUDA;
    float ms = 0.0f;
    if (cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) return GH_ERR_CUDA;
    tot += ms;
    ++n;
  }
  if (total_ms) *total_ms = tot;
  if (launches) *launches = n;
  return GH_OK;
}

int64_t gh_launch_count(void) { return launch_counter().load(); }

gh_status_t gh_debug_set(gh_debug_t knob, int64_t value) {
  switch (knob) {
    case GH_DEBUG_WAIT_LIMIT_NS: {
      const uint64_t v = value > 0 ? static_cast<uint64_t>(value) : kWaitTimeoutNs;
      if (cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v)) != cudaSuccess) return GH_ERR_CUDA;
      return GH_OK;
    }
    case GH_DEBUG_WITHHOLD_RING_PIECE:
      debug_ring_piece().store(value >= 0 ? value : -1);
      return GH_OK;
    case GH_DEBUG_WITHHOLD_GEMM_STAGE:
      debug_gemm_stage().store(value >= 0 && value < (int64_t(1) << 30) ? value : -1);
      return GH_OK;
  }
  return GH_ERR_INVALID_ARG;
}

const char* gh_status_string(gh_status_t s) {
  switch (s) {
    case GH_OK: return "ok";
    case GH_ERR_INVALID_ARG: return "invalid argument";
    case GH_ERR_UNSUPPORTED: return "unsupported";
    case GH_ERR_ALLOC: return "scratch allocation failed";
    case GH_ERR_CUDA: return "CUDA error";
    case GH_ERR_TIMEOUT: return "device wait timed out";
    case GH_ERR_TARGET_RANGE: return "target outside [0, V)";
  }
  return "unknown status";
}

const char* gh_version(void) { return "gh 0.1.0 sm_100a"; }

}  // extern "C"
