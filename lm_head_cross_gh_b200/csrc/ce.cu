// Standalone streaming cross-entropy, forward and backward in one call
// (Greyhound functional API, `cross_entropy`: "summed loss and logits
// gradient in one streaming pass"; nuvec FastOp::CrossEntropy /
// CrossEntropyVjp for the row loss and its gradient).
//
// Kernels, in launch order on the caller's stream:
//   ce_count_kernel  n_valid = #{t != ignore_index}; flags targets outside [0, V)
//   ce_row_kernel    one CTA (or a cluster of S CTAs) per row.  Each CTA pulls
//                    its slice of the row into shared memory with one bulk
//                    async copy per piece, folds an online (max, sum-exp) over
//                    it as the pieces land, exchanges the partial (max, sum)
//                    with its cluster peers through distributed shared memory,
//                    then rewrites the slice in place as the gradient and
//                    streams it back with a bulk async store.  HBM sees one
//                    read and one write of every logit.
//   ce_stream_kernel rows too long for the cluster path: two passes over
//                    global memory (the second one mostly from L2).
//   ce_reduce_kernel fixed-order (deterministic) sum of the per-row losses,
//                    divided by max(n_valid, 1) for "mean".
#include <algorithm>
#include <climits>
#include <cstdio>
#include <cstdlib>

#include "ce.h"
#include "common.cuh"
#include "profile.h"

namespace gh {

namespace {

template <typename T>
struct Elem;
template <>
struct Elem<float> {
  static constexpr int kBytes = 4;
  static __device__ __forceinline__ float load(const void* p) { return *reinterpret_cast<const float*>(p); }
  static __device__ __forceinline__ void store(void* p, float v) { *reinterpret_cast<float*>(p) = v; }
};
template <>
struct Elem<uint16_t> {  // bf16 bit pattern
  static constexpr int kBytes = 2;
  static __device__ __forceinline__ float load(const void* p) {
    return __uint_as_float(static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(p)) << 16);
  }
  static __device__ __forceinline__ void store(void* p, float v) {
    *reinterpret_cast<uint16_t*>(p) = to_bf16_bits(v);
  }
};

constexpr float kNegInf = -__builtin_huge_valf();

template <typename T>
__device__ __forceinline__ T neg_inf_elem();
template <>
__device__ __forceinline__ float neg_inf_elem<float>() { return kNegInf; }
template <>
__device__ __forceinline__ uint16_t neg_inf_elem<uint16_t>() { return 0xff80u; }

// Unpack one 16-byte chunk into floats.
template <typename T>
__device__ __forceinline__ void unpack16(const uint4& q, float (&v)[16 / Elem<T>::kBytes]);
template <>
__device__ __forceinline__ void unpack16<float>(const uint4& q, float (&v)[4]) {
  v[0] = __uint_as_float(q.x);
  v[1] = __uint_as_float(q.y);
  v[2] = __uint_as_float(q.z);
  v[3] = __uint_as_float(q.w);
}
template <>
__device__ __forceinline__ void unpack16<uint16_t>(const uint4& q, float (&v)[8]) {
  v[0] = bf16_lo(q.x); v[1] = bf16_hi(q.x);
  v[2] = bf16_lo(q.y); v[3] = bf16_hi(q.y);
  v[4] = bf16_lo(q.z); v[5] = bf16_hi(q.z);
  v[6] = bf16_lo(q.w); v[7] = bf16_hi(q.w);
}

template <typename T>
__device__ __forceinline__ uint4 pack16(const float (&g)[16 / Elem<T>::kBytes]);
template <>
__device__ __forceinline__ uint4 pack16<float>(const float (&g)[4]) {
  return make_uint4(__float_as_uint(g[0]), __float_as_uint(g[1]), __float_as_uint(g[2]), __float_as_uint(g[3]));
}
template <>
__device__ __forceinline__ uint4 pack16<uint16_t>(const float (&g)[8]) {
  return make_uint4(pack_bf16x2(g[0], g[1]), pack_bf16x2(g[2], g[3]), pack_bf16x2(g[4], g[5]),
                    pack_bf16x2(g[6], g[7]));
}

// Online (max, sum of exp(x - max)) state.  Combining is exact up to rounding
// and never forms (-inf) - (-inf).
struct MaxSum {
  float m, s;
};

__device__ __forceinline__ MaxSum combine(MaxSum a, MaxSum b) {
  const float M = fmaxf(a.m, b.m);
  if (M == kNegInf) return {kNegInf, 0.0f};
  const float sa = (a.m == kNegInf) ? 0.0f : a.s * ex2((a.m - M) * kLog2e);
  const float sb = (b.m == kNegInf) ? 0.0f : b.s * ex2((b.m - M) * kLog2e);
  return {M, sa + sb};
}

// Fold the 16/ES values of one chunk into the running state.
template <int N>
__device__ __forceinline__ void fold_chunk(MaxSum& st, const float (&v)[N]) {
  float cm = v[0];
#pragma unroll
  for (int i = 1; i < N; ++i) cm = fmaxf(cm, v[i]);
  if (cm == kNegInf) return;  // chunk of padding / -inf logits only
  if (cm > st.m) {
    st.s = (st.m == kNegInf) ? 0.0f : st.s * ex2((st.m - cm) * kLog2e);
    st.m = cm;
  }
  const float nm = -st.m * kLog2e;
  float acc = 0.0f;
#pragma unroll
  for (int i = 0; i < N; ++i) acc += ex2(fmaf(v[i], kLog2e, nm));
  st.s += acc;
}

__device__ __forceinline__ MaxSum warp_reduce(MaxSum st) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    MaxSum other{__shfl_xor_sync(0xffffffffu, st.m, o), __shfl_xor_sync(0xffffffffu, st.s, o)};
    st = combine(st, other);
  }
  return st;
}

// Block-wide reduction in a fixed order; every thread gets the result.
template <int kThreads>
__device__ __forceinline__ MaxSum block_reduce(MaxSum st, float* scratch /* 2*kWarps */) {
  constexpr int kWarps = kThreads / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  st = warp_reduce(st);
  if (lane == 0) {
    scratch[2 * warp] = st.m;
    scratch[2 * warp + 1] = st.s;
  }
  __syncthreads();
  MaxSum r{kNegInf, 0.0f};
#pragma unroll
  for (int w = 0; w < kWarps; ++w) r = combine(r, MaxSum{scratch[2 * w], scratch[2 * w + 1]});
  __syncthreads();
  return r;
}

// Block-wide max / sum; every thread gets the result.  `scratch` holds one
// float per warp and is not reused, so one barrier suffices.
template <int kThreads>
__device__ __forceinline__ float block_max(float v, float* scratch) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = scratch[0];
#pragma unroll
  for (int w = 1; w < kThreads / 32; ++w) r = fmaxf(r, scratch[w]);
  return r;
}

template <int kThreads>
__device__ __forceinline__ float block_sum(float v, float* scratch) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = scratch[0];
#pragma unroll
  for (int w = 1; w < kThreads / 32; ++w) r += scratch[w];
  return r;
}

template <int N>
__device__ __forceinline__ float tree_sum(const float (&e)[N]) {
  if constexpr (N == 8) {
    return ((e[0] + e[1]) + (e[2] + e[3])) + ((e[4] + e[5]) + (e[6] + e[7]));
  } else {
    return (e[0] + e[1]) + (e[2] + e[3]);
  }
}

__device__ __forceinline__ uint32_t bf16x2_max(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ uint4 pack_f16x8(const float (&e)[8]) {
  return make_uint4(pack_f16x2(e[0], e[1]), pack_f16x2(e[2], e[3]), pack_f16x2(e[4], e[5]),
                    pack_f16x2(e[6], e[7]));
}
template <int N>
__device__ __forceinline__ uint4 pack_f16x8(const float (&e)[N]) {  // fp32 rows keep their values
  return make_uint4(0, 0, 0, 0);
}

__device__ __forceinline__ float2 f16x2_to_f32(uint32_t w) {
  float lo, hi;
  asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(w));
  return make_float2(lo, hi);
}

template <int N>
__device__ __forceinline__ void unpack_f16x8(const uint4& q, float (&g)[N]) {
  const float2 a = f16x2_to_f32(q.x), b = f16x2_to_f32(q.y), c = f16x2_to_f32(q.z), d = f16x2_to_f32(q.w);
  g[0] = a.x; g[1] = a.y; g[2] = b.x; g[3] = b.y;
  if constexpr (N == 8) { g[4] = c.x; g[5] = c.y; g[6] = d.x; g[7] = d.y; }
}

constexpr int kMaxPieces = 4;
constexpr int kMinPieceChunks = 256;  // 4 KiB
constexpr int kRowThreads = 256;
constexpr int kStreamThreads = 1024;
constexpr int kHdrBytes = 128;        // barriers, cluster record, reduction scratch

struct RowShared {
  uint64_t bars[kMaxPieces];  // 32 B
  float rec_m, rec_s, rec_xt;  // partial published to the cluster
  int rec_has_t;
  float lse, xt;               // broadcast after the exchange
  float xt_local;              // target logit, when it lies in this CTA's slice
  float pad_;
  float red_m[kRowThreads / 32];
  float red_s[kRowThreads / 32];
};
static_assert(sizeof(RowShared) <= kHdrBytes, "header too large");

}  // namespace

__global__ void ce_count_kernel(const int64_t* __restrict__ t, int64_t n, int64_t V, int64_t ii,
                                unsigned long long* __restrict__ count) {
  unsigned long long c = 0;
  bool bad = false;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t v = t[i];
    if (v != ii) {
      if (v >= 0 && v < V) ++c;
      else bad = true;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0 && c) atomicAdd(count, c);
  if (bad) record_status(GH_ERR_TARGET_RANGE);
}

// One CTA per slice of `slice` elements; `cluster` CTAs per row (the launch's
// cluster dimension).  Dynamic shared memory: kHdrBytes + 16 * (chunks + 1).
//
// Chunk c of the slice buffer (16 bytes) is owned by thread c % kRowThreads in
// every pass, so the passes need no barrier between them apart from the two
// block reductions.  Passes, for a bf16 row:
//   0  max over the slice on packed bf16 pairs, piece by piece as copies land
//   1  e = 2^14 * exp(x - m) once per element: summed in fp32 and cached in
//      place as fp16 (the 2^14 keeps the cache in fp16's normal range down to
//      exp(x - m) = 2^-28)
//   2  gradient = k * e with one per-CTA factor k, stored straight to global
// For fp32 rows pass 1 only sums and pass 2 re-evaluates the exponent (the
// cache would not fit in place).
template <typename T>
__global__ void __launch_bounds__(kRowThreads) ce_row_kernel(CeArgs a) {
  constexpr int ES = Elem<T>::kBytes;
  constexpr int EPC = 16 / ES;
  constexpr bool kBf16 = ES == 2;
  constexpr float kShift = kBf16 ? 14.0f : 0.0f;  // log2 of the fp16 cache scale
  extern __shared__ __align__(128) uint8_t smem[];
  RowShared& sh = *reinterpret_cast<RowShared*>(smem);
  uint8_t* buf = smem + kHdrBytes;
  const int tid = threadIdx.x;

  const int S = a.cluster;
  const int64_t row = blockIdx.x / S;
  const int rank = static_cast<int>(blockIdx.x - row * S);
  const int64_t V = a.V;
  const int64_t e0 = static_cast<int64_t>(rank) * a.slice;
  const int n = static_cast<int>(tmax<int64_t>(0, tmin<int64_t>(V, e0 + a.slice) - e0));
  const int64_t t = a.targets[row];
  const bool valid = (t != a.ignore_index) && t >= 0 && t < V;

  const uint8_t* gsrc = reinterpret_cast<const uint8_t*>(a.logits) + (row * a.ld + e0) * ES;
  uint8_t* gdst = reinterpret_cast<uint8_t*>(a.grad) + (row * a.ld + e0) * ES;

  if (!valid) {
    // Ignored row: zero gradient, zero loss, no read of the logits.  Every CTA
    // of the cluster takes this branch, so no cluster barrier is entered.
    if (rank == 0 && tid == 0) a.row_loss[row] = 0.0f;
    const int glead = static_cast<int>(reinterpret_cast<uintptr_t>(gdst) & 15);
    const int gspan = glead + n * ES;
    const int c_lo = (glead + 15) >> 4, c_hi = max(c_lo, gspan >> 4);
    uint8_t* gbase = gdst - glead;
    for (int c = c_lo + tid; c < c_hi; c += kRowThreads)
      *reinterpret_cast<uint4*>(gbase + 16 * c) = make_uint4(0, 0, 0, 0);
    const int h = min(n, (16 * c_lo - glead) / ES);
    const int kt = max(h, (16 * c_hi - glead) / ES);
    for (int k = tid; k < h; k += kRowThreads) Elem<T>::store(gdst + k * ES, 0.0f);
    for (int k = kt + tid; k < n; k += kRowThreads) Elem<T>::store(gdst + k * ES, 0.0f);
    return;
  }

  // ---- issue the bulk loads ---------------------------------------------------------
  // buf byte j <-> global byte (gsrc - lead + j); element k at buf[lead + k*ES].
  const int lead = static_cast<int>(reinterpret_cast<uintptr_t>(gsrc) & 15);
  const int span = lead + n * ES;
  const int nchunks = (span + 15) >> 4;
  const int c_lo = (lead + 15) >> 4;       // first chunk fully inside the slice
  const int c_hi = max(c_lo, span >> 4);   // one past the last full chunk
  const int nbulk = c_hi - c_lo;
  const int npieces = nbulk == 0 ? 0 : max(1, min(kMaxPieces, nbulk / kMinPieceChunks));
  const uint8_t* gbase = gsrc - lead;

  if (tid == 0) {
    for (int p = 0; p < npieces; ++p) mbar_init(&sh.bars[p], 1);
    fence_mbar_init();
    for (int p = 0; p < npieces; ++p) {
      const int cs = c_lo + (nbulk * p) / npieces, ce = c_lo + (nbulk * (p + 1)) / npieces;
      const uint32_t bytes = 16u * (ce - cs);
      mbar_arrive_expect_tx(&sh.bars[p], bytes);
      bulk_g2s(buf + 16 * cs, gbase + 16 * cs, bytes, &sh.bars[p]);
    }
  }
  // The owners of the partial chunks at both ends fill them element by element
  // and pad them with -inf (which contributes exp(-inf) = 0 everywhere).
  auto fill_edge_chunk = [&](int c) {
    for (int b = 16 * c; b < 16 * c + 16; b += ES) {
      const int k = (b - lead) / ES;
      T v = neg_inf_elem<T>();
      if (b >= lead && k < n) v = *reinterpret_cast<const T*>(gsrc + k * ES);
      *reinterpret_cast<T*>(buf + b) = v;
    }
  };
  for (int c = tid; c < c_lo; c += kRowThreads) fill_edge_chunk(c);
  for (int c = c_hi + tid; c < nchunks; c += kRowThreads) fill_edge_chunk(c);
  __syncthreads();  // barriers initialised before anyone waits on them

  // ---- pass 0: max ---------------------------------------------------------------------
  bool ok = true;
  float m_thr;
  if constexpr (kBf16) {
    uint32_t mx = 0xff80ff80u;  // packed (-inf, -inf)
    auto fold_max = [&](int c) {
      const uint4 q = *reinterpret_cast<const uint4*>(buf + 16 * c);
      mx = bf16x2_max(mx, bf16x2_max(bf16x2_max(q.x, q.y), bf16x2_max(q.z, q.w)));
    };
    for (int c = tid; c < c_lo; c += kRowThreads) fold_max(c);
    for (int c = c_hi + tid; c < nchunks; c += kRowThreads) fold_max(c);
    for (int p = 0; p < npieces; ++p) {
      const int cs = c_lo + (nbulk * p) / npieces, ce = c_lo + (nbulk * (p + 1)) / npieces;
      if (!mbar_wait(&sh.bars[p], 0)) ok = false;
      int c = cs + ((tid - cs) % kRowThreads + kRowThreads) % kRowThreads;
      for (; c < ce; c += kRowThreads) fold_max(c);
    }
    m_thr = fmaxf(bf16_lo(mx), bf16_hi(mx));
  } else {
    m_thr = kNegInf;
    auto fold_max = [&](int c) {
      const float4 q = *reinterpret_cast<const float4*>(buf + 16 * c);
      m_thr = fmaxf(m_thr, fmaxf(fmaxf(q.x, q.y), fmaxf(q.z, q.w)));
    };
    for (int c = tid; c < c_lo; c += kRowThreads) fold_max(c);
    for (int c = c_hi + tid; c < nchunks; c += kRowThreads) fold_max(c);
    for (int p = 0; p < npieces; ++p) {
      const int cs = c_lo + (nbulk * p) / npieces, ce = c_lo + (nbulk * (p + 1)) / npieces;
      if (!mbar_wait(&sh.bars[p], 0)) ok = false;
      int c = cs + ((tid - cs) % kRowThreads + kRowThreads) % kRowThreads;
      for (; c < ce; c += kRowThreads) fold_max(c);
    }
  }
  const float m_cta = block_max<kRowThreads>(m_thr, sh.red_m);

  // ---- pass 1: sum of exp(x - m); bf16 rows cache 2^14 * exp(x - m) as fp16 ------------
  const int64_t tl = t - e0;  // target position within this slice
  const bool has_t = tl >= 0 && tl < n;
  const int tpos = has_t ? lead + static_cast<int>(tl) * ES : -1;  // byte position of the target
  // m_cta = -inf only for an empty slice; every exponent is then exp(-inf) = 0.
  const float nm = (m_cta == kNegInf) ? 0.0f : fmaf(-m_cta, kLog2e, kShift);
  float s_thr = 0.0f;
  for (int c = tid; c < nchunks; c += kRowThreads) {
    uint4* p = reinterpret_cast<uint4*>(buf + 16 * c);
    float v[EPC];
    unpack16<T>(*p, v);
    if ((tpos >> 4) == c) {
      const int ti = (tpos & 15) / ES;
#pragma unroll
      for (int i = 0; i < EPC; ++i)
        if (i == ti) sh.xt_local = v[i];
    }
    float e[EPC];
#pragma unroll
    for (int i = 0; i < EPC; ++i) e[i] = ex2(fmaf(v[i], kLog2e, nm));
    s_thr += tree_sum(e);
    if constexpr (kBf16) *p = pack_f16x8(e);
  }
  const float s_cta = block_sum<kRowThreads>(s_thr, sh.red_s) * (kBf16 ? (1.0f / 16384.0f) : 1.0f);

  // ---- combine across the cluster -----------------------------------------------------------
  float lse, xt;
  if (S == 1) {
    lse = m_cta + logf(s_cta);
    xt = sh.xt_local;
  } else {
    if (tid == 0) {
      sh.rec_m = m_cta;
      sh.rec_s = s_cta;
      sh.rec_has_t = has_t ? 1 : 0;
      sh.rec_xt = has_t ? sh.xt_local : 0.0f;
    }
    cluster_arrive_release();
    cluster_wait_acquire();
    if (tid == 0) {
      MaxSum tot{kNegInf, 0.0f};
      float x = 0.0f;
      for (int r = 0; r < S; ++r) {  // fixed rank order: identical on every CTA
        MaxSum pr{ld_dsmem_f32(map_to_rank(&sh.rec_m, r)), ld_dsmem_f32(map_to_rank(&sh.rec_s, r))};
        tot = combine(tot, pr);
        if (ld_dsmem_s32(map_to_rank(&sh.rec_has_t, r))) x = ld_dsmem_f32(map_to_rank(&sh.rec_xt, r));
      }
      sh.lse = tot.m + logf(tot.s);
      sh.xt = x;
    }
    cluster_arrive_release();  // this CTA is done reading its peers
    __syncthreads();
    lse = sh.lse;
    xt = sh.xt;
  }
  if (rank == 0 && tid == 0) a.row_loss[row] = (lse - xt) + a.z * lse * lse;

  // ---- pass 2: gradient straight to global ----------------------------------------------------
  const unsigned long long nv = *a.n_valid;
  const float scale = a.mean ? 1.0f / static_cast<float>(nv > 0 ? nv : 1ull) : 1.0f;
  const float coef = scale * (1.0f + 2.0f * a.z * lse);
  // bf16: g = coef * exp(x - lse) = k * (2^14 exp(x - m)), k = coef * 2^-14 * exp(m - lse)
  // fp32: g = coef * 2^(x log2e - lse log2e)
  const float k = (m_cta == kNegInf) ? 0.0f : coef * ex2(fmaf(m_cta - lse, kLog2e, -kShift));
  const float nl = -lse * kLog2e;
  uint8_t* dbase = gdst - lead;
  if (ok) {
    for (int c = tid; c < nchunks; c += kRowThreads) {
      const uint4 q = *reinterpret_cast<const uint4*>(buf + 16 * c);
      float g[EPC];
      if constexpr (kBf16) {
        unpack_f16x8(q, g);
#pragma unroll
        for (int i = 0; i < EPC; ++i) g[i] *= k;
      } else {
        float v[EPC];
        unpack16<T>(q, v);
#pragma unroll
        for (int i = 0; i < EPC; ++i) g[i] = coef * ex2(fmaf(v[i], kLog2e, nl));
      }
      if ((tpos >> 4) == c) {
        const int ti = (tpos & 15) / ES;
#pragma unroll
        for (int i = 0; i < EPC; ++i)
          if (i == ti) g[i] -= scale;
      }
      if (a.congruent && c >= c_lo && c < c_hi) {
        *reinterpret_cast<uint4*>(dbase + 16 * c) = pack16<T>(g);
      } else {
#pragma unroll
        for (int i = 0; i < EPC; ++i) {
          const int kk = (16 * c + i * ES - lead) / ES;
          if (16 * c + i * ES >= lead && kk < n) Elem<T>::store(gdst + kk * ES, g[i]);
        }
      }
    }
  }
  if (S > 1) cluster_wait_acquire();  // peers have finished reading this CTA's record
}

// Rows too long for the shared-memory path: one CTA per row, two passes over
// global memory.  Element loads/stores are scalar at the row's unaligned ends.
template <typename T>
__global__ void __launch_bounds__(kStreamThreads) ce_stream_kernel(CeArgs a) {
  constexpr int ES = Elem<T>::kBytes;
  constexpr int EPC = 16 / ES;
  __shared__ float red[2 * (kStreamThreads / 32)];
  const int tid = threadIdx.x;
  const int64_t row = blockIdx.x;
  const int64_t V = a.V;
  const int64_t t = a.targets[row];
  const bool valid = (t != a.ignore_index) && t >= 0 && t < V;
  const uint8_t* src = reinterpret_cast<const uint8_t*>(a.logits) + row * a.ld * ES;
  uint8_t* dst = reinterpret_cast<uint8_t*>(a.grad) + row * a.ld * ES;

  const int lead = static_cast<int>(reinterpret_cast<uintptr_t>(src) & 15);
  const int64_t span = lead + V * ES;
  const int64_t c_lo = (lead + 15) >> 4;
  const int64_t c_hi = tmax<int64_t>(c_lo, span >> 4);
  const int64_t h = tmin<int64_t>(V, (16 * c_lo - lead) / ES);
  const int64_t kt = tmax<int64_t>(h, (16 * c_hi - lead) / ES);
  const uint8_t* sbase = src - lead;

  if (!valid) {
    if (tid == 0) a.row_loss[row] = 0.0f;
    for (int64_t k = tid; k < V; k += kStreamThreads) Elem<T>::store(dst + k * ES, 0.0f);
    return;
  }
  MaxSum st{kNegInf, 0.0f};
  for (int64_t c = c_lo + tid; c < c_hi; c += kStreamThreads) {
    const uint4 q = *reinterpret_cast<const uint4*>(sbase + 16 * c);
    float v[EPC];
    unpack16<T>(q, v);
    fold_chunk(st, v);
  }
  for (int64_t k = tid; k < h; k += kStreamThreads) {
    float v[1] = {Elem<T>::load(src + k * ES)};
    fold_chunk(st, v);
  }
  for (int64_t k = kt + tid; k < V; k += kStreamThreads) {
    float v[1] = {Elem<T>::load(src + k * ES)};
    fold_chunk(st, v);
  }
  st = block_reduce<kStreamThreads>(st, red);
  const float lse = st.m + logf(st.s);
  const float xt = Elem<T>::load(src + t * ES);
  if (tid == 0) a.row_loss[row] = (lse - xt) + a.z * lse * lse;

  const unsigned long long nv = *a.n_valid;
  const float scale = a.mean ? 1.0f / static_cast<float>(nv > 0 ? nv : 1ull) : 1.0f;
  const float coef = scale * (1.0f + 2.0f * a.z * lse);
  const float nl = -lse * kLog2e;
  auto gval = [&](float x, int64_t k) {
    float g = coef * ex2(fmaf(x, kLog2e, nl));
    return k == t ? g - scale : g;
  };
  if (a.congruent) {
    uint8_t* dbase = dst - lead;
    for (int64_t c = c_lo + tid; c < c_hi; c += kStreamThreads) {
      const uint4 q = *reinterpret_cast<const uint4*>(sbase + 16 * c);
      float v[EPC], g[EPC];
      unpack16<T>(q, v);
      const int64_t k0 = (16 * c - lead) / ES;
#pragma unroll
      for (int i = 0; i < EPC; ++i) g[i] = gval(v[i], k0 + i);
      *reinterpret_cast<uint4*>(dbase + 16 * c) = pack16<T>(g);
    }
    for (int64_t k = tid; k < h; k += kStreamThreads) Elem<T>::store(dst + k * ES, gval(Elem<T>::load(src + k * ES), k));
    for (int64_t k = kt + tid; k < V; k += kStreamThreads)
      Elem<T>::store(dst + k * ES, gval(Elem<T>::load(src + k * ES), k));
  } else {
    for (int64_t k = tid; k < V; k += kStreamThreads) Elem<T>::store(dst + k * ES, gval(Elem<T>::load(src + k * ES), k));
  }
}

// Deterministic sum of the row losses (fixed per-thread stride, fixed tree),
// accumulated in double, then the reduction's division.
__global__ void __launch_bounds__(1024) ce_reduce_kernel(const float* __restrict__ row_loss, int64_t B,
                                                         const unsigned long long* __restrict__ n_valid,
                                                         int mean, float* __restrict__ loss) {
  __shared__ double red[32];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < B; i += 1024) s += static_cast<double>(row_loss[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double tot = 0.0;
    for (int w = 0; w < 32; ++w) tot += red[w];
    if (mean) {
      const unsigned long long nv = *n_valid;
      tot /= static_cast<double>(nv > 0 ? nv : 1ull);
    }
    *loss = static_cast<float>(tot);
  }
}

// ------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------

static int ce_max_slice_bytes() {
  // Slices up to 64 KiB keep three or more row-CTAs resident per SM.
  static int v = [] {
    const char* e = std::getenv("GH_CE_SLICE_KB");
    int kb = e ? std::atoi(e) : 64;
    return std::min(std::max(kb, 4), 200) * 1024;
  }();
  return v;
}

CePlan ce_plan(int64_t V, int elem_bytes) {
  CePlan p{};
  const int64_t max_slice = ce_max_slice_bytes();
  int S = 1;
  auto slice_for = [&](int s) {
    int64_t q = (V + s - 1) / s;
    return ((q + 15) / 16) * 16;  // slices start on 32/64-byte boundaries of the row
  };
  while (S < 8 && slice_for(S) * elem_bytes > max_slice) S *= 2;
  int64_t q = slice_for(S);
  if (q * elem_bytes > 200 * 1024) {
    p.streaming = true;
    p.cluster = 1;
    p.slice = 0;
    p.smem_bytes = 0;
    return p;
  }
  p.streaming = false;
  p.cluster = S;
  p.slice = static_cast<int>(q);
  const int64_t chunks = (15 + q * elem_bytes + 15) / 16 + 1;
  p.smem_bytes = static_cast<int>(kHdrBytes + 16 * chunks);
  return p;
}

gh_status_t ce_launch(const CeArgs& args_in, int64_t B, gh_dtype_t dtype, cudaStream_t stream) {
  CeArgs a = args_in;
  const int es = dtype == GH_F32 ? 4 : 2;
  const CePlan plan = ce_plan(a.V, es);
  a.cluster = plan.cluster;
  a.slice = plan.slice;

  if (B * plan.cluster > INT32_MAX) return GH_ERR_UNSUPPORTED;  // one grid covers every row
  if (plan.streaming) {
    ProfileScope prof(GH_KERNEL_CE_ROW, stream);
    if (dtype == GH_F32) ce_stream_kernel<float><<<static_cast<unsigned>(B), kStreamThreads, 0, stream>>>(a);
    else ce_stream_kernel<uint16_t><<<static_cast<unsigned>(B), kStreamThreads, 0, stream>>>(a);
    note_launch();
    return cudaGetLastError() == cudaSuccess ? GH_OK : GH_ERR_CUDA;
  }

  void (*kern)(CeArgs) = dtype == GH_F32 ? ce_row_kernel<float> : ce_row_kernel<uint16_t>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, plan.smem_bytes) != cudaSuccess)
    return GH_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(B * plan.cluster));
  cfg.blockDim = dim3(kRowThreads);
  cfg.dynamicSmemBytes = plan.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = plan.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  ProfileScope prof(GH_KERNEL_CE_ROW, stream);
  note_launch();
  if (cudaLaunchKernelEx(&cfg, kern, a) != cudaSuccess) return GH_ERR_CUDA;
  return GH_OK;
}

gh_status_t ce_count_launch(const int64_t* targets, int64_t n, int64_t V, int64_t ii,
                            unsigned long long* count, cudaStream_t stream) {
  if (cudaMemsetAsync(count, 0, sizeof(unsigned long long), stream) != cudaSuccess) return GH_ERR_CUDA;
  if (n == 0) return GH_OK;
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, 148 * 4);
  ce_count_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(targets, n, V, ii, count);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? GH_OK : GH_ERR_CUDA;
}

gh_status_t ce_reduce_launch(const float* row_loss, int64_t B, const unsigned long long* n_valid, int mean,
                             float* loss, cudaStream_t stream) {
  ce_reduce_kernel<<<1, 1024, 0, stream>>>(row_loss, B, n_valid, mean, loss);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? GH_OK : GH_ERR_CUDA;
}

}  // namespace gh
