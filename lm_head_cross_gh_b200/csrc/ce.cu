// Standalone cross-entropy, forward and backward in one call (Greyhound
// functional API, `cross_entropy`: the summed or mean loss and the logits
// gradient from one call; nuvec FastOp::CrossEntropy / CrossEntropyVjp for the
// row loss and its gradient).  The ring pipelines in ce_ring.cu take batches
// of 8 rows per SM or more; the row kernel below takes the smaller ones.
//
// Kernels, in launch order on the caller's stream:
//   ce_count_kernel  n_valid = #{t != ignore_index}; flags targets outside [0, V)
//   ce_row_kernel    persistent; one CTA (or a cluster of S CTAs) per row at a
//                    time.  Each CTA pulls its slice of a row into one of two
//                    shared-memory buffers with a bulk async copy (the next
//                    rows' copies are in flight while a row is computed), takes
//                    the max, caches exp(x - max) once per element, exchanges
//                    partial (max, sum) with its cluster peers through
//                    distributed shared memory, and stores the gradient
//                    straight to global.  HBM sees one read and one write of
//                    every logit.
//   ce_stream_kernel rows too long for the cluster path: two passes over
//                    global memory (the second one mostly from L2).
//   ce_reduce_kernel fixed-order (deterministic) sum of the per-row losses,
//                    divided by max(n_valid, 1) for "mean".
#include <algorithm>
#include <climits>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include <cuda_fp16.h>

#include "ce.h"
#include "ce_device.cuh"
#include "common.cuh"
#include "profile.h"

namespace gh {

namespace {


#ifndef GH_CE_ROW_THREADS
#define GH_CE_ROW_THREADS 512
#endif
constexpr int kRowThreads = GH_CE_ROW_THREADS;  // two row groups of half this size
#ifndef GH_CE_UNROLL
#define GH_CE_UNROLL 4
#endif
constexpr int kUnroll = GH_CE_UNROLL;  // chunks a thread handles per loop iteration
constexpr int kStreamThreads = 1024;
constexpr int kPieces = 4;                     // bulk copies (and barriers) per slice
constexpr int kMinPieceChunks = 256;           // 4 KiB
constexpr int kHdrBytes = 1024;                // barriers, targets, records, reduction scratch
constexpr int kMaxSliceBytes = 110 * 1024;     // two slice buffers per CTA fit in 227 KiB
constexpr int kMaxCluster = 8;

struct RowShared {
  uint64_t full[2][kPieces];                   // load barriers of the two groups' buffers
  uint64_t xbar[2][2];                         // per group, per valid-row parity: cluster records in
  int64_t tgt[2][2];                           // per group: targets of its next two rows
  float4 xrec[2][2][kMaxCluster];              // per group, per parity, per rank: (m, s, xt, has_t)
  float lse[2], xt[2], xt_local[2];            // per group, broadcast within the group
  float pad_[2];
  float red_m[kRowThreads / 32];
  float red_s[kRowThreads / 32];
};
static_assert(sizeof(RowShared) <= kHdrBytes, "header too large");

// Geometry of one CTA's slice of one row: elements [e0, e0 + n) at global
// address gsrc.  Slice buffer byte j <-> global byte (gsrc - lead + j).
// Chunks [c_lo, c_hi) are whole 16-byte chunks inside the slice; the chunks
// before and after hold the ragged ends.  Chunks [x_lo, x_hi) are copied in
// bulk: the ragged-end chunks too, whenever their 16 bytes lie inside the
// logits buffer (the bytes outside the slice are then overwritten with -inf).
struct SliceGeo {
  const uint8_t* gsrc;
  uint8_t* gdst;
  int n, lead, span, nchunks, c_lo, c_hi, x_lo, x_hi;
};

template <int ES>
__device__ __forceinline__ SliceGeo slice_geo(const CeArgs& a, int64_t row, int rank) {
  SliceGeo g;
  const int64_t e0 = static_cast<int64_t>(rank) * a.slice;
  g.n = static_cast<int>(tmax<int64_t>(0, tmin<int64_t>(a.V, e0 + a.slice) - e0));
  g.gsrc = reinterpret_cast<const uint8_t*>(a.logits) + (row * a.ld + e0) * ES;
  g.gdst = reinterpret_cast<uint8_t*>(a.grad) + (row * a.ld + e0) * ES;
  g.lead = static_cast<int>(reinterpret_cast<uintptr_t>(g.gsrc) & 15);
  g.span = g.lead + g.n * ES;
  g.nchunks = (g.span + 15) >> 4;
  g.c_lo = (g.lead + 15) >> 4;
  g.c_hi = max(g.c_lo, g.span >> 4);
  const uint8_t* lo_bound = reinterpret_cast<const uint8_t*>(a.logits);
  const uint8_t* hi_bound = lo_bound + a.B * a.ld * ES;
  const uint8_t* gbase = g.gsrc - g.lead;
  g.x_lo = (g.n > 0 && gbase >= lo_bound) ? 0 : g.c_lo;
  g.x_hi = (g.n > 0 && gbase + 16 * g.nchunks <= hi_bound) ? g.nchunks : g.c_hi;
  if (g.x_hi < g.x_lo) g.x_hi = g.x_lo;
  return g;
}

__device__ __forceinline__ bool target_valid(const CeArgs& a, int64_t t) {
  return (t != a.ignore_index) && t >= 0 && t < a.V;
}


// Group leader: start the bulk copies of this CTA's slice of `row` into `buf`.
// Every valid row arrives on all a.npieces barriers of the buffer (the piece
// count is fixed per launch, so the barriers' phases stay in step however the
// rows' alignment varies); a piece with no bytes completes on the arrive alone.
template <int ES>
__device__ __forceinline__ void issue_slice(const CeArgs& a, int64_t row, int64_t t, int rank, uint8_t* buf,
                                            uint64_t* bars) {
  if (row >= a.B || !target_valid(a, t)) return;
  const SliceGeo g = slice_geo<ES>(a, row, rank);
  const int nb = g.x_hi - g.x_lo;
  const int np = a.npieces;
  const uint8_t* gbase = g.gsrc - g.lead;
  for (int p = 0; p < np; ++p) {
    const int cs = g.x_lo + (nb * p) / np, ce = g.x_lo + (nb * (p + 1)) / np;
    const uint32_t bytes = 16u * (ce - cs);
    mbar_arrive_expect_tx(&bars[p], bytes);
    if (bytes) bulk_g2s(buf + 16 * cs, gbase + 16 * cs, bytes, &bars[p]);
  }
}

}  // namespace

__global__ void ce_count_kernel(const int64_t* __restrict__ t, int64_t n, int64_t V, int64_t ii,
                                unsigned long long* __restrict__ count) {
  pdl_wait();
  pdl_trigger();
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

// Single-CTA count for batches up to 2^20 rows: no atomics, no prior memset.
__global__ void __launch_bounds__(1024) ce_count1_kernel(const int64_t* __restrict__ t, int64_t n, int64_t V,
                                                         int64_t ii, unsigned long long* __restrict__ count) {
  __shared__ unsigned long long part[32];
  pdl_wait();
  pdl_trigger();
  unsigned long long c = 0;
  bool bad = false;
  for (int64_t i = threadIdx.x; i < n; i += 1024) {
    const int64_t v = t[i];
    if (v != ii) {
      if (v >= 0 && v < V) ++c;
      else bad = true;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = c;
  if (bad) record_status(GH_ERR_TARGET_RANGE);
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long tot = 0;
    for (int w = 0; w < 32; ++w) tot += part[w];
    *count = tot;
  }
}

// Persistent row kernel.  A CTA holds NG independent row groups of
// kRowThreads / NG threads.  With NG = 2 (rows of one slice) each group owns
// one slice buffer and its own rows; the two groups drift out of phase, so one
// group's exponent pass overlaps the other's loads and stores.  With NG = 1 a
// cluster of `cluster` CTAs shares each row (one slice each) and every CTA
// double-buffers its slices.  A buffer's bulk copy is split into pieces with
// one barrier each, so work starts as soon as the first piece lands.
//
// Chunk c (16 bytes) of a slice belongs to thread c % (group size) in every
// pass, so the passes of a row need no barrier between them; each thread works
// relative to the max m_t of its own chunks.  For a bf16 row:
//   0  m_t = max over the thread's chunks, on packed bf16 pairs
//   1  e = 2^14 exp(x - m_t) once per element: summed in fp32 and cached in
//      place as fp16 (the 2^14 keeps the cache in fp16's normal range down to
//      exp(x - m_t) = 2^-28)
//   *  one group combine of (m_t, s_t); the CTAs of a cluster exchange (max,
//      sum, target logit) once through distributed shared memory
//   2  gradient = k_t e, k_t = scale (1 + 2 z lse) 2^-14 exp(m_t - lse),
//      stored straight to global; the target element is rewritten by its
//      owner afterwards with the -scale term.
// fp32 rows only sum in pass 1 and re-evaluate the exponent in pass 2 (a
// cache would not fit in place).
template <typename T, int MODE>
__global__ void __launch_bounds__(kRowThreads, 1) ce_row_kernel(CeArgs a) {
  constexpr int NG = 2;                 // row groups per CTA
  constexpr int ES = Elem<T>::kBytes;
  constexpr int EPC = 16 / ES;
  constexpr int NT = kRowThreads / NG;  // threads per group
  constexpr int GW = NT / 32;           // warps per group
  constexpr bool kBf16 = ES == 2;
  constexpr float kShift = kBf16 ? 14.0f : 0.0f;  // log2 of the fp16 cache scale
  extern __shared__ __align__(128) uint8_t smem[];
  RowShared& sh = *reinterpret_cast<RowShared*>(smem);
  const int grp = NG == 1 ? 0 : static_cast<int>(threadIdx.x) / NT;
  const int tid = static_cast<int>(threadIdx.x) - grp * NT;  // thread within the group
  const int lane = tid & 31, gwarp = tid >> 5;
  const bool leader = tid == 0;
  const int S = a.cluster;
  const int cid = blockIdx.x / S;
  const int rank = blockIdx.x - cid * S;
  const int64_t ngroups = static_cast<int64_t>(gridDim.x / S) * NG;
  const int64_t first = static_cast<int64_t>(cid) * NG + grp;
  auto gsync = [&]() { asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "r"(NT) : "memory"); };
  auto slot_of = [&](int64_t) { return grp; };
  auto buf_of = [&](int slot) { return smem + kHdrBytes + slot * a.buf_bytes; };
  auto row_of = [&](int64_t k) { return first + k * ngroups; };
  auto tgt_of = [&](int64_t k) { return row_of(k) < a.B ? a.targets[row_of(k)] : int64_t(0); };

  if (threadIdx.x == 0) {
    for (int sl = 0; sl < 2; ++sl) {
      for (int p = 0; p < kPieces; ++p) mbar_init(&sh.full[sl][p], 1);
      mbar_init(&sh.xbar[sl][0], S);
      mbar_init(&sh.xbar[sl][1], S);
    }
    fence_mbar_init();
  }
  pdl_wait();     // the predecessor's outputs (targets, logits, counter) are complete
  pdl_trigger();  // persistent grid: every CTA is resident, the next kernel may start launching
  if (leader) {
    sh.tgt[grp][0] = tgt_of(0);
    sh.tgt[grp][1] = tgt_of(1);
  }
  __syncthreads();
  if (S > 1) {  // every CTA's exchange barriers are initialised before any peer arrives on them
    cluster_arrive_release();
    cluster_wait_acquire();
  }
  if (leader) issue_slice<ES>(a, row_of(0), sh.tgt[grp][0], rank, buf_of(grp), sh.full[grp]);

  uint32_t phase = 0;       // bit sl: parity of the next waits on slot sl
  uint32_t valid_rows = 0;  // selects the exchange barrier and record buffer
  uint32_t xphase = 0;      // bit pb: parity of the next wait on xbar[grp][pb]
  bool ok = true;
  constexpr bool with_grad = MODE == kModeFwdBwd;
  const unsigned long long nv = with_grad ? *a.n_valid : 1ull;
  const float scale = a.mean ? 1.0f / static_cast<float>(nv > 0 ? nv : 1ull) : 1.0f;

  for (int64_t k = 0; row_of(k) < a.B; ++k) {
    const int64_t row = row_of(k);
    const int sl = slot_of(k);
    uint8_t* buf = buf_of(sl);
    const int64_t t = sh.tgt[grp][k & 1];
    // the leader fetches the target of row k + 2 early; it is stored after this row
    const int64_t t_ahead = leader ? tgt_of(k + 2) : 0;
    const SliceGeo g = slice_geo<ES>(a, row, rank);

    if (!target_valid(a, t)) {
      // Ignored row: zero gradient, zero loss, the logits are never read.  An
      // out-of-range index of the selective log-softmax gives NaN.
      if (rank == 0 && leader) {
        if constexpr (MODE == kModeSelect) {
          a.row_loss[row] = __int_as_float(0x7fc00000);
          record_status(GH_ERR_TARGET_RANGE);
        } else {
          a.row_loss[row] = 0.0f;
        }
      }
      if constexpr (with_grad) {
      const int glead = static_cast<int>(reinterpret_cast<uintptr_t>(g.gdst) & 15);
      const int gspan = glead + g.n * ES;
      const int z_lo = (glead + 15) >> 4, z_hi = max(z_lo, gspan >> 4);
      uint8_t* zb = g.gdst - glead;
      for (int c = z_lo + tid; c < z_hi; c += NT) *reinterpret_cast<uint4*>(zb + 16 * c) = make_uint4(0, 0, 0, 0);
      const int h = min(g.n, (16 * z_lo - glead) / ES);
      const int kt = max(h, (16 * z_hi - glead) / ES);
      for (int e = tid; e < h; e += NT) Elem<T>::store(g.gdst + e * ES, 0.0f);
      for (int e = kt + tid; e < g.n; e += NT) Elem<T>::store(g.gdst + e * ES, 0.0f);
      }
    } else {
      // ---- pass 0: this thread's max, piece by piece as copies land ----------------------
      const int nb = g.x_hi - g.x_lo;
      const int np = a.npieces;
      // ragged ends outside the bulk range: element loads by their owners
      auto fill_edge = [&](int c) {
        for (int bb = 16 * c; bb < 16 * c + 16; bb += ES) {
          const int e = (bb - g.lead) / ES;
          T v = neg_inf_elem<T>();
          if (bb >= g.lead && e < g.n) v = *reinterpret_cast<const T*>(g.gsrc + e * ES);
          *reinterpret_cast<T*>(buf + bb) = v;
        }
      };
      uint32_t mx0 = 0xff80ff80u, mx1 = 0xff80ff80u;  // bf16: packed (-inf, -inf)
      float mf = kNegInf;                              // fp32
      auto fold_max = [&](int c) {
        const uint4 q = *reinterpret_cast<const uint4*>(buf + 16 * c);
        if constexpr (kBf16) {
          mx0 = bf16x2_max(mx0, bf16x2_max(bf16x2_max(q.x, q.y), bf16x2_max(q.z, q.w)));
        } else {
          mf = fmaxf(mf, fmaxf(fmaxf(__uint_as_float(q.x), __uint_as_float(q.y)),
                               fmaxf(__uint_as_float(q.z), __uint_as_float(q.w))));
        }
      };
      for (int c = tid; c < g.x_lo; c += NT) {
        fill_edge(c);
        fold_max(c);
      }
      for (int c = g.x_hi + ((tid - g.x_hi) % NT + NT) % NT; c < g.nchunks; c += NT) {
        fill_edge(c);
        fold_max(c);
      }
      for (int p = 0; p < np; ++p) {
        const int cs = g.x_lo + (nb * p) / np, ce = g.x_lo + (nb * (p + 1)) / np;
        if (!mbar_wait(&sh.full[sl][p], (phase >> sl) & 1)) ok = false;
        // bulk-copied ragged ends: overwrite the bytes outside the slice with -inf
        if (p == 0 && g.x_lo == 0 && g.lead > 0 && tid == 0)
          for (int bb = 0; bb < g.lead; bb += ES) *reinterpret_cast<T*>(buf + bb) = neg_inf_elem<T>();
        if (p == np - 1 && g.x_hi == g.nchunks && (g.span & 15) && tid == (g.nchunks - 1) % NT)
          for (int bb = g.span; bb < 16 * g.nchunks; bb += ES) *reinterpret_cast<T*>(buf + bb) = neg_inf_elem<T>();
        int c = cs + ((tid - cs) % NT + NT) % NT;
        for (; c + (kUnroll - 1) * NT < ce; c += kUnroll * NT) {
          uint4 q[kUnroll];
#pragma unroll
          for (int u = 0; u < kUnroll; ++u) q[u] = *reinterpret_cast<const uint4*>(buf + 16 * (c + u * NT));
#pragma unroll
          for (int u = 0; u < kUnroll; ++u) {
            if constexpr (kBf16) {
              uint32_t& m = (u & 1) ? mx1 : mx0;
              m = bf16x2_max(m, bf16x2_max(bf16x2_max(q[u].x, q[u].y), bf16x2_max(q[u].z, q[u].w)));
            } else {
              mf = fmaxf(mf, fmaxf(fmaxf(__uint_as_float(q[u].x), __uint_as_float(q[u].y)),
                                   fmaxf(__uint_as_float(q[u].z), __uint_as_float(q[u].w))));
            }
          }
        }
        for (; c < ce; c += NT) fold_max(c);
      }
      phase ^= 1u << sl;  // every valid row completes one phase on each piece barrier
      float m_t;
      if constexpr (kBf16) {
        mx0 = bf16x2_max(mx0, mx1);
        m_t = fmaxf(bf16_lo(mx0), bf16_hi(mx0));
      } else {
        m_t = mf;
      }

      // ---- target logit (its owner reads it before pass 1 overwrites the chunk) -----------
      const int64_t tl = t - static_cast<int64_t>(rank) * a.slice;  // target position in this slice
      const bool has_t = tl >= 0 && tl < g.n;
      const int tpos = has_t ? g.lead + static_cast<int>(tl) * ES : -1;
      const bool own_t = has_t && ((tpos >> 4) % NT) == tid;
      if (own_t) sh.xt_local[grp] = Elem<T>::load(buf + tpos);

      // ---- pass 1: sum of exp(x - m_t); bf16 rows cache 2^14 exp(x - m_t) as fp16 --------
      const float nm = (m_t == kNegInf) ? 0.0f : fmaf(-m_t, kLog2e, kShift);
      float s_t;
      {
        const float2 l2 = make_float2(kLog2e, kLog2e), nm2 = make_float2(nm, nm);
        float2 acc = make_float2(0.0f, 0.0f);
        auto exps = [&](const uint4& q, float (&e)[EPC]) {
          float v[EPC];
          unpack16<T>(q, v);
#pragma unroll
          for (int j = 0; j < EPC; j += 2) {
            const float2 y = __ffma2_rn(make_float2(v[j], v[j + 1]), l2, nm2);
            e[j] = ex2(y.x);
            e[j + 1] = ex2(y.y);
          }
#pragma unroll
          for (int j = 0; j < EPC; j += 2) acc = __fadd2_rn(acc, make_float2(e[j], e[j + 1]));
        };
        int c = tid;
        for (; c + (kUnroll - 1) * NT < g.nchunks; c += kUnroll * NT) {
          uint4 q[kUnroll];
#pragma unroll
          for (int u = 0; u < kUnroll; ++u) q[u] = *reinterpret_cast<const uint4*>(buf + 16 * (c + u * NT));
#pragma unroll
          for (int u = 0; u < kUnroll; ++u) {
            float e[EPC];
            exps(q[u], e);
            if (kBf16 && with_grad) *reinterpret_cast<uint4*>(buf + 16 * (c + u * NT)) = pack_f16x8(e);
          }
        }
        for (; c < g.nchunks; c += NT) {
          uint4* p0 = reinterpret_cast<uint4*>(buf + 16 * c);
          float e0[EPC];
          exps(*p0, e0);
          if (kBf16 && with_grad) *p0 = pack_f16x8(e0);
        }
        s_t = acc.x + acc.y;
      }

      // ---- combine (m_t, s_t) over the group, then over the cluster ------------------------
      MaxSum ms{m_t, s_t};
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        MaxSum other{__shfl_xor_sync(0xffffffffu, ms.m, o), __shfl_xor_sync(0xffffffffu, ms.s, o)};
        ms = combine(ms, other);
      }
      float* red_m = sh.red_m + grp * GW;
      float* red_s = sh.red_s + grp * GW;
      if (lane == 0) {
        red_m[gwarp] = ms.m;
        red_s[gwarp] = ms.s;
      }
      gsync();
      const int pb = valid_rows & 1;
      if (gwarp == 0) {
        MaxSum w = lane < GW ? MaxSum{red_m[lane], red_s[lane]} : MaxSum{kNegInf, 0.0f};
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          MaxSum other{__shfl_xor_sync(0xffffffffu, w.m, o), __shfl_xor_sync(0xffffffffu, w.s, o)};
          w = combine(w, other);
        }
        if (lane == 0) {
          const float s_cta = w.s * (kBf16 ? (1.0f / 16384.0f) : 1.0f);
          if (S == 1) {
            sh.lse[grp] = w.m + logf(s_cta);
            sh.xt[grp] = sh.xt_local[grp];
          } else {
            // Publish this slice's (max, sum, target logit) into every rank's
            // record slot `rank` and arrive on its barrier for this row parity;
            // then wait for all ranks' records here and combine them in rank
            // order (the same lse on every CTA).
            const float xtv = has_t ? sh.xt_local[grp] : 0.0f;
            for (int q = 0; q < S; ++q) {
              st_dsmem_v4(map_to_rank(&sh.xrec[grp][pb][rank], q), w.m, s_cta, xtv, has_t ? 1.0f : 0.0f);
              mbar_arrive_cluster(map_to_rank(&sh.xbar[grp][pb], q));
            }
            if (!mbar_wait_cluster(&sh.xbar[grp][pb], (xphase >> pb) & 1)) ok = false;
            MaxSum tot{kNegInf, 0.0f};
            float x = 0.0f;
            for (int q = 0; q < S; ++q) {
              const float4 r = sh.xrec[grp][pb][q];
              tot = combine(tot, MaxSum{r.x, r.y});
              if (r.w != 0.0f) x = r.z;
            }
            sh.lse[grp] = tot.m + logf(tot.s);
            sh.xt[grp] = x;
          }
        }
      }
      if (S > 1) xphase ^= 1u << pb;
      gsync();
      const float lse = sh.lse[grp];
      ++valid_rows;
      if (rank == 0 && leader)
        a.row_loss[row] = MODE == kModeSelect ? sh.xt[grp] - lse : (lse - sh.xt[grp]) + a.z * lse * lse;

      // ---- pass 2: gradient straight to global -------------------------------------------
      const float coef = scale * (1.0f + 2.0f * a.z * lse);
      const float k_t = (m_t == kNegInf) ? 0.0f : coef * ex2(fmaf(m_t - lse, kLog2e, -kShift));
      const float nl = -lse * kLog2e;
      const float2 k2 = make_float2(k_t, k_t);
      auto grad16 = [&](const uint4& q, float (&gv)[EPC]) {
        if constexpr (kBf16) {
          float e[EPC];
          unpack_f16x8(q, e);
#pragma unroll
          for (int j = 0; j < EPC; j += 2) {
            const float2 r = __fmul2_rn(make_float2(e[j], e[j + 1]), k2);
            gv[j] = r.x;
            gv[j + 1] = r.y;
          }
        } else {
          float v[EPC];
          unpack16<T>(q, v);
#pragma unroll
          for (int j = 0; j < EPC; ++j) gv[j] = coef * ex2(fmaf(v[j], kLog2e, nl));
        }
      };
      auto store_elems = [&](int c, const float (&gv)[EPC]) {
#pragma unroll
        for (int j = 0; j < EPC; ++j) {
          const int e = (16 * c + j * ES - g.lead) / ES;
          if (16 * c + j * ES >= g.lead && e < g.n) Elem<T>::store(g.gdst + e * ES, gv[j]);
        }
      };
      if (ok && with_grad) {
        if (a.congruent) {
          uint8_t* dbase = g.gdst - g.lead;
          int c = g.c_lo + ((tid - g.c_lo) % NT + NT) % NT;
          for (; c + (kUnroll - 1) * NT < g.c_hi; c += kUnroll * NT) {
            uint4 q[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) q[u] = *reinterpret_cast<const uint4*>(buf + 16 * (c + u * NT));
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
              float g0[EPC];
              grad16(q[u], g0);
              *reinterpret_cast<uint4*>(dbase + 16 * (c + u * NT)) = pack16<T>(g0);
            }
          }
          for (; c < g.c_hi; c += NT) {
            const uint4 q0 = *reinterpret_cast<const uint4*>(buf + 16 * c);
            float g0[EPC];
            grad16(q0, g0);
            *reinterpret_cast<uint4*>(dbase + 16 * c) = pack16<T>(g0);
          }
          for (int ce = tid; ce < g.c_lo; ce += NT) {
            float g0[EPC];
            grad16(*reinterpret_cast<const uint4*>(buf + 16 * ce), g0);
            store_elems(ce, g0);
          }
          for (int ce = g.c_hi + ((tid - g.c_hi) % NT + NT) % NT; ce < g.nchunks; ce += NT) {
            float g0[EPC];
            grad16(*reinterpret_cast<const uint4*>(buf + 16 * ce), g0);
            store_elems(ce, g0);
          }
        } else {
          for (int c = tid; c < g.nchunks; c += NT) {
            float g0[EPC];
            grad16(*reinterpret_cast<const uint4*>(buf + 16 * c), g0);
            store_elems(c, g0);
          }
        }
        if (own_t) {  // the target element, rewritten after its chunk with the -scale term
          float gt;
          if constexpr (kBf16) {
            gt = k_t * f16_to_f32(*reinterpret_cast<const uint16_t*>(buf + tpos));
          } else {
            gt = coef * ex2(fmaf(sh.xt_local[grp], kLog2e, nl));
          }
          Elem<T>::store(g.gdst + tl * ES, gt - scale);
        }
      }
    }
    // The buffer is free once every thread of the group is past this row; its
    // generic-proxy writes are ordered before the bulk copy that refills it.
    fence_proxy_async_smem();
    gsync();
    if (leader) {
      sh.tgt[grp][k & 1] = t_ahead;  // row k + 2's target (row k + 1's is already stored)
      issue_slice<ES>(a, row_of(k + 1), sh.tgt[grp][(k + 1) & 1], rank, buf, sh.full[sl]);
    }
  }
  // No peer writes into this CTA after its last row: every rank's last records
  // for this CTA were waited for above.
}

// Rows too long for the shared-memory path: one CTA per row, two passes over
// global memory.  Element loads/stores are scalar at the row's unaligned ends.
template <typename T, int MODE>
__global__ void __launch_bounds__(kStreamThreads) ce_stream_kernel(CeArgs a) {
  constexpr int ES = Elem<T>::kBytes;
  constexpr int EPC = 16 / ES;
  __shared__ float red[2 * (kStreamThreads / 32)];
  pdl_wait();
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

  constexpr bool with_grad = MODE == kModeFwdBwd;
  if (!valid) {
    if (tid == 0) {
      if constexpr (MODE == kModeSelect) {
        a.row_loss[row] = __int_as_float(0x7fc00000);
        record_status(GH_ERR_TARGET_RANGE);
      } else {
        a.row_loss[row] = 0.0f;
      }
    }
    if (with_grad)
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
  if (tid == 0) a.row_loss[row] = MODE == kModeSelect ? xt - lse : (lse - xt) + a.z * lse * lse;
  if constexpr (!with_grad) return;

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
  pdl_wait();
  pdl_trigger();
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

static int ce_slice_target_bytes() {
  // Largest slice before a row is split across a cluster (tunable for sweeps).
  static int v = [] {
    const char* e = std::getenv("GH_CE_SLICE_KB");
    const int kb = e ? std::atoi(e) : 110;
    return std::min(std::max(kb, 4), kMaxSliceBytes / 1024) * 1024;
  }();
  return v;
}

// Plan for rows of V elements split over a cluster of S CTAs.
static CePlan plan_for_cluster(int64_t V, int elem_bytes, int S) {
  CePlan p{};
  int64_t q = (V + S - 1) / S;
  q = ((q + 15) / 16) * 16;  // slices start on 32/64-byte boundaries of the row
  if (q * elem_bytes > kMaxSliceBytes) {
    p.streaming = true;
    p.cluster = 1;
    return p;
  }
  p.streaming = false;
  p.cluster = S;
  p.slice = static_cast<int>(q);
  const int64_t chunks = (15 + q * elem_bytes + 15) / 16 + 1;
  p.buf_bytes = static_cast<int>(((16 * chunks) + 127) / 128 * 128);
  p.smem_bytes = kHdrBytes + 2 * p.buf_bytes;
  return p;
}

// The smallest cluster whose slices fit the slice target (a launch may still
// pick a larger one that keeps more SMs busy: see row_plan).
CePlan ce_plan(int64_t V, int elem_bytes) {
  const int64_t target = ce_slice_target_bytes();
  int S = 1;
  while (S < kMaxCluster && ((V + S - 1) / S + 15) / 16 * 16 * elem_bytes > target) ++S;
  return plan_for_cluster(V, elem_bytes, S);
}

static int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

namespace {

using CeKernel = void (*)(CeArgs);

template <typename T>
CeKernel row_kernel_mode(int mode) {
  return mode == kModeSelect ? ce_row_kernel<T, kModeSelect>
         : mode == kModeFwd  ? ce_row_kernel<T, kModeFwd>
                             : ce_row_kernel<T, kModeFwdBwd>;
}
CeKernel row_kernel_for(int es, int mode) {
  return es == 4 ? row_kernel_mode<float>(mode) : row_kernel_mode<uint16_t>(mode);
}
template <typename T>
CeKernel stream_kernel_mode(int mode) {
  return mode == kModeSelect ? ce_stream_kernel<T, kModeSelect>
         : mode == kModeFwd  ? ce_stream_kernel<T, kModeFwd>
                             : ce_stream_kernel<T, kModeFwdBwd>;
}

// Launch plan of the row kernel for one (device, V, element size), computed
// once: the occupancy queries and attribute calls cost far more than a launch.
struct PlanEntry {
  int dev;
  int64_t V;
  int es;
  CePlan plan;
  int64_t active;  // resident clusters
};

std::mutex g_plan_mu;
PlanEntry g_plans[64];
int g_nplans = 0;

gh_status_t row_plan(int64_t V, int es, CePlan* out, int64_t* active_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GH_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_plan_mu);
  for (int i = 0; i < g_nplans; ++i) {
    if (g_plans[i].dev == dev && g_plans[i].V == V && g_plans[i].es == es) {
      *out = g_plans[i].plan;
      *active_out = g_plans[i].active;
      return GH_OK;
    }
  }
  CePlan plan = ce_plan(V, es);
  int64_t active = 0;
  if (!plan.streaming) {
    CeKernel kern = row_kernel_for(es, kModeFwdBwd);
    // The dynamic shared memory limit is an attribute of the kernel, shared by
    // every plan: raise it once per device to the opt-in maximum, for the
    // kernel of every mode (they share one launch plan).
    static bool raised[64][2] = {};
    const int kv = es == 4;
    if (dev < 64 && !raised[dev][kv]) {
      int optin = 0;
      if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return GH_ERR_CUDA;
      for (int m : {kModeFwdBwd, kModeFwd, kModeSelect})
        if (cudaFuncSetAttribute(row_kernel_for(es, m), cudaFuncAttributeMaxDynamicSharedMemorySize, optin) !=
            cudaSuccess)
          return GH_ERR_CUDA;
      raised[dev][kv] = true;
    }
    // Clusters must fit inside a GPC, so the number resident at once depends on
    // the cluster size.  (A larger cluster that keeps more SMs busy measured
    // slower: 262144-vocab rows, 6 CTAs x 22 clusters 1.22 ms vs 5 x 26 1.11 ms.)
    auto resident = [&](const CePlan& pl) -> int64_t {
      cudaLaunchConfig_t cfg = {};
      cfg.blockDim = dim3(kRowThreads);
      cfg.dynamicSmemBytes = pl.smem_bytes;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = pl.cluster;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      cfg.gridDim = dim3(static_cast<unsigned>(pl.cluster * device_sm_count()));
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        n = 0;
      }
      return n;
    };
    active = resident(plan);
    if (plan.smem_bytes > kHdrBytes + 2 * (kMaxSliceBytes + 256)) return GH_ERR_UNSUPPORTED;
    if (active <= 0) return GH_ERR_UNSUPPORTED;
  }
  if (std::getenv("GH_DEBUG_PLAN"))
    std::fprintf(stderr, "gh ce plan: V=%lld es=%d streaming=%d cluster=%d slice=%d buf=%d smem=%d clusters=%lld\n",
                 static_cast<long long>(V), es, plan.streaming ? 1 : 0, plan.cluster, plan.slice, plan.buf_bytes,
                 plan.smem_bytes, static_cast<long long>(active));
  if (g_nplans < 64) g_plans[g_nplans++] = PlanEntry{dev, V, es, plan, active};
  *out = plan;
  *active_out = active;
  return GH_OK;
}

}  // namespace

// Rows take the ring pipelines (ce_ring.cu) when there are enough of them to
// keep every SM's ring busy (round-robin rows: at least kRingMinRowsPerSm per
// SM keeps the last wave's imbalance small); fewer rows take the row kernel,
// whose clusters split long rows over several SMs.  GH_CE_PATH=ring or =rows
// forces one of the two (tests, measurements).
constexpr int kRingMinRowsPerSm = 8;

static bool use_ring(int64_t B, int sms) {
  const char* e = std::getenv("GH_CE_PATH");
  if (e && std::strcmp(e, "ring") == 0) return true;
  if (e && std::strcmp(e, "rows") == 0) return false;
  return B >= static_cast<int64_t>(kRingMinRowsPerSm) * sms;
}

gh_status_t ce_launch(const CeArgs& args_in, int64_t B, gh_dtype_t dtype, cudaStream_t stream) {
  CeArgs a = args_in;
  a.B = B;
  const int es = dtype == GH_F32 ? 4 : 2;
  {
    const int sms = device_sm_count();
    if (use_ring(B, sms)) return ce_ring_launch(a, es, static_cast<int>(std::min<int64_t>(B, sms)), stream);
  }
  CePlan plan;
  int64_t active = 0;
  gh_status_t st = row_plan(a.V, es, &plan, &active);
  if (st != GH_OK) return st;
  a.cluster = plan.cluster;
  a.slice = plan.slice;
  a.buf_bytes = plan.buf_bytes;
  a.npieces = std::max(1, std::min(kPieces, (plan.slice * es / 16) / kMinPieceChunks));

  if (plan.streaming) {
    if (B > INT32_MAX) return GH_ERR_UNSUPPORTED;
    ProfileScope prof(a.profile_kind, stream);
    const CeKernel sk = es == 4 ? stream_kernel_mode<float>(a.mode) : stream_kernel_mode<uint16_t>(a.mode);
    const cudaError_t e = launch_pdl(sk, dim3(static_cast<unsigned>(B)), dim3(kStreamThreads), 0, stream, 1, a);
    note_launch();
    return e == cudaSuccess ? GH_OK : GH_ERR_CUDA;
  }

  const CeKernel kern = row_kernel_for(es, a.mode);
  // Persistent grid: as many clusters as can be resident at once, no more
  // than there are rows (two per cluster, one per row group).
  const int64_t nclusters = std::min<int64_t>(active, (B + 1) / 2);
  ProfileScope prof(a.profile_kind, stream);
  note_launch();
  if (launch_pdl(kern, dim3(static_cast<unsigned>(nclusters * plan.cluster)), dim3(kRowThreads), plan.smem_bytes,
                 stream, plan.cluster, a) != cudaSuccess)
    return GH_ERR_CUDA;
  return GH_OK;
}

gh_status_t ce_count_launch(const int64_t* targets, int64_t n, int64_t V, int64_t ii,
                            unsigned long long* count, cudaStream_t stream) {
  if (n <= (int64_t(1) << 20)) {
    // one CTA counts without atomics and writes the counter itself
    const cudaError_t e = launch_pdl(ce_count1_kernel, dim3(1), dim3(1024), 0, stream, 1, targets, n, V, ii, count);
    note_launch();
    return e == cudaSuccess ? GH_OK : GH_ERR_CUDA;
  }
  if (cudaMemsetAsync(count, 0, sizeof(unsigned long long), stream) != cudaSuccess) return GH_ERR_CUDA;
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, 148 * 4);
  const cudaError_t e =
      launch_pdl(ce_count_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream, 1, targets, n, V, ii, count);
  note_launch();
  return e == cudaSuccess ? GH_OK : GH_ERR_CUDA;
}

gh_status_t ce_reduce_launch(const float* row_loss, int64_t B, const unsigned long long* n_valid, int mean,
                             float* loss, cudaStream_t stream) {
  const cudaError_t e = launch_pdl(ce_reduce_kernel, dim3(1), dim3(1024), 0, stream, 1, row_loss, B, n_valid, mean, loss);
  note_launch();
  return e == cudaSuccess ? GH_OK : GH_ERR_CUDA;
}

}  // namespace gh
