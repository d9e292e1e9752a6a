// Device helpers shared by the cross-entropy kernels (ce.cu, ce_ring.cu):
// element access for fp32 and bf16 rows, 16-byte chunk (un)packing, and the
// online (max, sum of exponentials) state with its exact-up-to-rounding merge.
#pragma once

#include <cstdint>
#include <cstring>

#include <cuda_fp16.h>

#include "common.cuh"

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
  __half2 h;
  memcpy(&h, &w, sizeof(h));
  return __half22float2(h);
}

__device__ __forceinline__ float f16_to_f32(uint16_t h) {
  float f;
  asm("{\n\t.reg .f16 x;\n\tmov.b16 x, %1;\n\tcvt.f32.f16 %0, x;\n\t}" : "=f"(f) : "h"(h));
  return f;
}

template <int N>
__device__ __forceinline__ void unpack_f16x8(const uint4& q, float (&g)[N]) {
  const float2 a = f16x2_to_f32(q.x), b = f16x2_to_f32(q.y), c = f16x2_to_f32(q.z), d = f16x2_to_f32(q.w);
  g[0] = a.x; g[1] = a.y; g[2] = b.x; g[3] = b.y;
  if constexpr (N == 8) { g[4] = c.x; g[5] = c.y; g[6] = d.x; g[7] = d.y; }
}

}  // namespace
}  // namespace gh
