// gh_ce_fwd_bwd_noalloc: the standalone cross-entropy for callers that cannot
// allocate device memory during a call.
//
// gh_ce_fwd_bwd takes its scratch (the valid-token counter and one float per
// row) from cudaMallocAsync on the caller's stream.  Some callers cannot do
// that: a runtime whose device memory is already reserved in full by another
// allocator (a framework's caching allocator, a fixed arena planned ahead of
// time) would see the allocation fail mid-step, and latency-critical loops
// that forbid any allocator call inside a step cannot use it either.  This
// variant takes its scratch from a fixed array in the library's own device
// image instead and allocates nothing.
//
// The array lives in every GPU that loads the library until the process
// exits.  Its device address is looked up once per device (on the first call
// made with that device current) and cached.  All calls share the one array:
// calls whose work overlaps on the GPU (different streams, or different host
// threads) race on it and must be serialised by the caller.
#include <cmath>
#include <mutex>

#include "ce.h"
#include "common.cuh"

namespace gh {
namespace {

// Scratch: the valid-token counter (256 bytes reserved) followed by one float
// per row.
constexpr int64_t kNoAllocMaxRows = 65536;
constexpr size_t kNoAllocScratchBytes = 256 + sizeof(float) * kNoAllocMaxRows;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device.  In host code
// the symbol is only a host-side stand-in, so it must never be passed to a
// kernel directly; cudaGetSymbolAddress gives the real device address.
gh_status_t noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GH_ERR_CUDA;
  std::lock_guard<std::mutex> g(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      (void)cudaGetLastError();
      return GH_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return GH_OK;
}

}  // namespace
}  // namespace gh

extern "C" gh_status_t gh_ce_fwd_bwd_noalloc(const void* logits, const int64_t* targets, int64_t B, int64_t V,
                                             gh_dtype_t dtype, int64_t ignore_index, gh_reduction_t reduction,
                                             float z_mult, float* loss, void* grad, void* stream_) {
  using namespace gh;
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
    const uintptr_t l0 = reinterpret_cast<uintptr_t>(logits), g0 = reinterpret_cast<uintptr_t>(grad);
    const uintptr_t bytes = static_cast<uintptr_t>(B) * static_cast<uintptr_t>(V) * es;
    if (l0 < g0 + bytes && g0 < l0 + bytes) return GH_ERR_INVALID_ARG;
  }
  // The fixed scratch holds one float per row for at most kNoAllocMaxRows rows.
  if (B > kNoAllocMaxRows) return GH_ERR_UNSUPPORTED;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (B == 0) return cudaMemsetAsync(loss, 0, sizeof(float), stream) == cudaSuccess ? GH_OK : GH_ERR_CUDA;

  void* scratch = nullptr;
  gh_status_t st = noalloc_scratch(&scratch);
  if (st != GH_OK) return st;
  // The array keeps the previous call's contents: ce_count_launch overwrites
  // the counter (a kernel store or a memset, never an allocation) and the row
  // kernel writes every row's loss slot before the reduction reads it.
  unsigned long long* n_valid = static_cast<unsigned long long*>(scratch);
  float* row_loss = reinterpret_cast<float*>(static_cast<char*>(scratch) + 256);

  const int mean = reduction == GH_REDUCTION_MEAN;
  st = ce_count_launch(targets, B, V, ignore_index, n_valid, stream);
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
  return st;
}
