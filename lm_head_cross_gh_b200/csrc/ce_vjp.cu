// Vector-Jacobian product of the per-row cross-entropy (nuvec
// FastOp::CrossEntropyVjp: logits, targets, the forward's row loss and an
// upstream gradient g per row give the logits gradient).
//
// The forward's row loss is lse - x_t, so lse = loss + x_t comes back from one
// element of the row and no reduction is needed: the gradient
//     grad_j = g (exp(x_j - lse) - [j == t])
// takes one read and one write of every logit, in a single sweep per row.  Rows
// whose target equals ignore_index (or lies outside [0, V)) get a zero row.
//
// ce_vjp_kernel: persistent CTAs of 512 threads, rows round-robin.  Thread 0
// loads the row's target, loss and g (and the target logit) into shared memory
// one row ahead; the row's whole 16-byte chunks go through registers four at a
// time (16-byte loads, `st.global.cs` 16-byte stores when the gradient row has
// the logits row's 16-byte phase), the ragged ends element by element.
#include "ce.h"
#include "ce_device.cuh"
#include "common.cuh"
#include "profile.h"

namespace gh {

namespace {

constexpr int kVjpThreads = 512;
constexpr int kVjpUnroll = 4;

struct VjpRow {
  int64_t row;
  float g, nl;  // upstream gradient, -lse log2(e)
  int64_t t;    // target (-1: zero row)
};

template <typename T>
__device__ __forceinline__ void vjp_chunk(const uint4& q, float g, float nl, int tj, uint8_t* dst, bool congruent) {
  constexpr int EPC = 16 / Elem<T>::kBytes;
  constexpr int ES = Elem<T>::kBytes;
  float v[EPC], r[EPC];
  unpack16<T>(q, v);
  const float2 l2 = make_float2(kLog2e, kLog2e), nl2 = make_float2(nl, nl), g2 = make_float2(g, g);
#pragma unroll
  for (int j = 0; j < EPC; j += 2) {
    const float2 y = __ffma2_rn(make_float2(v[j], v[j + 1]), l2, nl2);
    const float2 e = __fmul2_rn(make_float2(ex2(y.x), ex2(y.y)), g2);
    r[j] = e.x;
    r[j + 1] = e.y;
  }
  if (tj >= 0) {
#pragma unroll
    for (int j = 0; j < EPC; ++j)
      if (j == tj) r[j] -= g;
  }
  if (congruent) {
    __stcs(reinterpret_cast<uint4*>(dst), pack16<T>(r));
  } else {
#pragma unroll
    for (int j = 0; j < EPC; ++j) Elem<T>::store(dst + j * ES, r[j]);
  }
}

template <typename T>
__global__ void __launch_bounds__(kVjpThreads) ce_vjp_kernel(const void* __restrict__ logits, const int64_t* targets,
                                                             const float* row_loss, const float* gup, void* grad,
                                                             int64_t B, int64_t V, int64_t ii, int congruent) {
  constexpr int ES = Elem<T>::kBytes;
  __shared__ VjpRow info[2];
  pdl_wait();
  pdl_trigger();
  const int tid = static_cast<int>(threadIdx.x);
  const int64_t G = gridDim.x;
  // thread 0 fetches row `row`'s scalars into info[slot]
  auto fetch = [&](int64_t row, int slot) {
    VjpRow w{row, 0.0f, 0.0f, -1};
    if (row < B) {
      const int64_t t = targets[row];
      if (t != ii && t >= 0 && t < V) {
        const float xt = Elem<T>::load(static_cast<const uint8_t*>(logits) + (row * V + t) * ES);
        const float lse = row_loss[row] + xt;
        w.g = gup[row];
        w.nl = -lse * kLog2e;
        w.t = t;
      } else if (t != ii) {
        record_status(GH_ERR_TARGET_RANGE);
      }
    }
    info[slot] = w;
  };
  if (tid == 0) fetch(blockIdx.x, 0);
  int slot = 0;
  for (int64_t row = blockIdx.x; row < B; row += G, slot ^= 1) {
    // info[slot] is written (prologue or the previous row) and every thread is
    // done with info[slot ^ 1], which thread 0 then refills for the next row
    __syncthreads();
    const VjpRow w = info[slot];
    if (tid == 0) fetch(row + G, slot ^ 1);
    const uint8_t* src = static_cast<const uint8_t*>(logits) + row * V * ES;
    uint8_t* dst = static_cast<uint8_t*>(grad) + row * V * ES;
    const int lead = static_cast<int>(reinterpret_cast<uintptr_t>(src) & 15);
    const int64_t span = lead + V * ES;
    const int64_t c_lo = (lead + 15) >> 4, c_hi = tmax<int64_t>(c_lo, span >> 4);
    const int64_t h = tmin<int64_t>(V, (16 * c_lo - lead) / ES);
    const int64_t tail = tmax<int64_t>(h, (16 * c_hi - lead) / ES);
    const uint8_t* sbase = src - lead;
    uint8_t* gbase = dst - lead;  // chunk c's gradient bytes start at gbase + 16 c
    if (w.t < 0) {  // zero row
      if (congruent) {
        for (int64_t c = c_lo + tid; c < c_hi; c += kVjpThreads)
          __stcs(reinterpret_cast<uint4*>(gbase + 16 * c), make_uint4(0, 0, 0, 0));
      } else {
        for (int64_t e = h + tid; e < tail; e += kVjpThreads) Elem<T>::store(dst + e * ES, 0.0f);
      }
      if (tid < h) Elem<T>::store(dst + static_cast<int64_t>(tid) * ES, 0.0f);
      if (tid >= 32 && tid < 48 && tail + (tid - 32) < V) Elem<T>::store(dst + (tail + (tid - 32)) * ES, 0.0f);
      continue;
    }
    const int64_t tb = lead + w.t * ES;  // target byte in the row's chunk space
    const int64_t tc = tb >> 4;
    const int tj = static_cast<int>((tb & 15) / ES);
    const bool cg = congruent != 0;
    int64_t c = c_lo + tid;
    for (; c + (kVjpUnroll - 1) * kVjpThreads < c_hi; c += kVjpUnroll * kVjpThreads) {
      uint4 q[kVjpUnroll];
#pragma unroll
      for (int u = 0; u < kVjpUnroll; ++u)
        q[u] = __ldcg(reinterpret_cast<const uint4*>(sbase + 16 * (c + u * kVjpThreads)));
#pragma unroll
      for (int u = 0; u < kVjpUnroll; ++u) {
        const int64_t cu = c + u * kVjpThreads;
        vjp_chunk<T>(q[u], w.g, w.nl, cu == tc ? tj : -1, gbase + 16 * cu, cg);
      }
    }
    for (; c < c_hi; c += kVjpThreads)
      vjp_chunk<T>(__ldcg(reinterpret_cast<const uint4*>(sbase + 16 * c)), w.g, w.nl, c == tc ? tj : -1,
                   gbase + 16 * c, cg);
    // ragged ends: threads 0-15 the head elements, 32-47 the tail
    int64_t e = -1;
    if (tid < h) e = tid;
    if (tid >= 32 && tid < 48 && tail + (tid - 32) < V) e = tail + (tid - 32);
    if (e >= 0) {
      const float x = Elem<T>::load(src + e * ES);
      float r = w.g * ex2(fmaf(x, kLog2e, w.nl));
      if (e == w.t) r -= w.g;
      Elem<T>::store(dst + e * ES, r);
    }
  }
}

}  // namespace

gh_status_t ce_vjp_launch(const void* logits, const int64_t* targets, const float* row_loss, const float* g,
                          void* grad, int64_t B, int64_t V, int64_t ignore_index, gh_dtype_t dtype,
                          cudaStream_t stream) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) (void)cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t grid = tmin<int64_t>(B, static_cast<int64_t>(sms) * 4);
  const int congruent =
      ((reinterpret_cast<uintptr_t>(logits) ^ reinterpret_cast<uintptr_t>(grad)) & 15) == 0 ? 1 : 0;
  ProfileScope prof(GH_KERNEL_CE_VJP, stream);
  note_launch();
  const cudaError_t e =
      dtype == GH_F32
          ? launch_pdl(ce_vjp_kernel<float>, dim3(static_cast<unsigned>(grid)), dim3(kVjpThreads), 0, stream, 1,
                       logits, targets, row_loss, g, grad, B, V, ignore_index, congruent)
          : launch_pdl(ce_vjp_kernel<uint16_t>, dim3(static_cast<unsigned>(grid)), dim3(kVjpThreads), 0, stream, 1,
                       logits, targets, row_loss, g, grad, B, V, ignore_index, congruent);
  return e == cudaSuccess ? GH_OK : GH_ERR_CUDA;
}

}  // namespace gh
