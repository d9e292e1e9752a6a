// Cross-entropy rows as one streaming pipeline per SM: the forward-only kernel
// (the loss without its gradient, and the selective log-softmax x[index] -
// lse) and, further down, the two-pass forward+backward kernel built on it.
//
// Nothing has to stay in shared memory once it has been read, so instead of
// a whole row resident in shared memory (the row kernel in ce.cu) a ring of
// fixed-size pieces runs across row boundaries:
//
//   warp 16 (producer)   walks this CTA's rows and their pieces in order and
//                        starts a bulk copy into the next free ring slot;
//   warps 0-15 (consumers, four groups of four warps)
//                        piece n goes whole to group n % 4: as it lands, each
//                        thread loads its eight chunks into registers, the
//                        group frees the slot at once, and the thread folds the
//                        chunks into its online (max, sum of exp) state;
//                        at a row's end each thread posts its state to the
//                        row's finalizer (no reduction on the consumers);
//   warps 17-20 (finalizers)
//                        take the valid rows in turn (row k to warp 17 + k % 4);
//                        each merges the 512 thread states with the row's ragged
//                        ends (the elements outside the whole 16-byte chunks,
//                        read from global), reads the target logit and writes
//                        the row value.  With four of them, a finalizer's
//                        global loads for a row have about four rows' time
//                        to arrive before the row's states do.
//
// Every logit is read from HBM once and every element costs one exponential;
// the consumers never wait on each other, and the producer stays up to
// kRingSlots pieces (192 KiB) ahead.  Rows are assigned round-robin to the
// persistent CTAs; all barriers are mbarriers with bounded waits.
#include "ce.h"
#include "ce_device.cuh"
#include "common.cuh"
#include "profile.h"

namespace gh {

namespace {

constexpr int kRingConsumerWarps = 16;
constexpr int kRingConsumers = 32 * kRingConsumerWarps;
// The consumers form kRingGroups groups; piece n goes to group n % kRingGroups
// whole, so each group's warps (one per SM sub-partition) run out of phase
// with the other groups' and one group's loads and max overlap another's
// exponentials.
constexpr int kRingGroups = 4;
constexpr int kGroupWarps = kRingConsumerWarps / kRingGroups;
constexpr int kGroupThreads = 32 * kGroupWarps;
constexpr int kRingFinalizers = 4;                 // warps; also the row-state buffers in flight
constexpr int kRingThreads = kRingConsumers + 32 + 32 * kRingFinalizers;  // + producer warp
constexpr int kRingSlots = 12;
constexpr int kRingPieceBytes = 16384;
constexpr int kRingPieceChunks = kRingPieceBytes / 16;
constexpr int kPieceChunksPerThread = kRingPieceChunks / kGroupThreads;  // 8
static_assert(kRingSlots % kRingGroups == 0, "a slot always serves the same group");
static_assert(kRingPieceChunks % kGroupThreads == 0, "whole chunks per thread");
constexpr int kRingHdrBytes = 17408;  // barriers, 4 x 512 row states, lse

struct RingShared {
  uint64_t full[kRingSlots];   // piece landed (producer's expect_tx + the copy's bytes)
  uint64_t empty[kRingSlots];  // piece consumed (one arrival per warp of its group)
  uint64_t rowfull[kRingFinalizers];   // per valid row k % 4: every consumer warp posted its state
  uint64_t rowempty[kRingFinalizers];  // per valid row k % 4: its finalizer has read the states
  uint64_t lseready[kRingFinalizers];  // two-pass kernel, per valid row k % 4: lse[k % 4] is set
  float2 part[kRingFinalizers][kRingConsumerWarps][32];  // every consumer thread's row state
  float lse[kRingFinalizers];
  int abort;                   // a wait ran out: every role stops waiting
};
static_assert(sizeof(RingShared) <= kRingHdrBytes, "ring header too large");

// Byte geometry of one row: chunks [c_lo, c_hi) (16-byte, counted from the
// row's first byte rounded down to 16) lie wholly inside the row and are
// copied in bulk; the h head elements [0, h) and the tail elements [tail, V)
// are the ragged ends, read element by element.
struct RingRow {
  const uint8_t* base;  // row start rounded down to 16 bytes
  int c_lo, c_hi, h, tail;
};

template <int ES>
__device__ __forceinline__ RingRow ring_row(const CeArgs& a, int64_t row) {
  RingRow r;
  const uint8_t* src = static_cast<const uint8_t*>(a.logits) + row * a.ld * ES;
  const int lead = static_cast<int>(reinterpret_cast<uintptr_t>(src) & 15);
  const int64_t span = lead + a.V * ES;
  r.base = src - lead;
  r.c_lo = (lead + 15) >> 4;
  r.c_hi = static_cast<int>(tmax<int64_t>(r.c_lo, span >> 4));
  r.h = static_cast<int>(tmin<int64_t>(a.V, (16 * r.c_lo - lead) / ES));
  r.tail = static_cast<int>(tmax<int64_t>(r.h, (16 * static_cast<int64_t>(r.c_hi) - lead) / ES));
  return r;
}

__device__ __forceinline__ int ring_pieces(const RingRow& r) {
  return (r.c_hi - r.c_lo + kRingPieceChunks - 1) / kRingPieceChunks;
}

__device__ __forceinline__ bool ring_target_valid(const CeArgs& a, int64_t t) {
  return (t != a.ignore_index) && t >= 0 && t < a.V;
}

// A finalizer lane's share of a row's merge: the states consumer lane `lane`
// of each of the 16 consumer warps posted (max first, then one rescale each).
__device__ __forceinline__ MaxSum merge_lane_states(const float2 (*part)[32], int lane) {
  float m[kRingConsumerWarps], sv[kRingConsumerWarps];
  float M = kNegInf;
#pragma unroll
  for (int w = 0; w < kRingConsumerWarps; ++w) {
    const float2 v = part[w][lane];
    m[w] = v.x;
    sv[w] = v.y;
    M = fmaxf(M, v.x);
  }
  if (M == kNegInf) return {kNegInf, 0.0f};
  float S = 0.0f;
#pragma unroll
  for (int w = 0; w < kRingConsumerWarps; ++w)
    if (m[w] != kNegInf) S += sv[w] * ex2((m[w] - M) * kLog2e);
  return {M, S};
}

// The running reference of a thread's online sum is its max so far plus
// kRingBump: a rescale happens only when a chunk beats the reference, so a row
// whose values keep creeping upwards rescales once per kRingBump of growth
// instead of once per chunk (each rescale costs an approximate exponential's
// rounding).  Terms then sit at or below exp(-kRingBump); fp32 keeps every term
// within ~79 of the max, and the rest are below 1e-34 of the sum.
constexpr float kRingBump = 8.0f;

__device__ __forceinline__ void raise_ref(MaxSum& st, float cm) {
  if (cm > st.m) {
    const float mn = cm + kRingBump;
    st.s = (st.m == kNegInf) ? 0.0f : st.s * ex2((st.m - mn) * kLog2e);
    st.m = mn;
  }
}

// 2^y on the FMA pipe for y <= 0 (the MUFU unit is the busiest pipe of the
// ring; pass 1 sends part of its exponentials here): y is clamped at -125
// (max.NaN: a NaN stays NaN), split Cody-Waite style into r = round(y) (the
// 1.5 * 2^23 rounding constant leaves r in the low mantissa bits) and
// f = y - r in [-0.5, 0.5]; 2^f comes from a degree-5 polynomial
// (coefficients fitted here to the relative error of 2^f on that interval:
// 2.3e-7 in fp32 Horner form), multiplied by 2^r built in the exponent field
// (exact: r >= -125 keeps both factors and the product normal, and a NaN
// argument makes a NaN product, as ex2.approx does).
__device__ __forceinline__ float max_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

__device__ __forceinline__ float2 exp2_fma2(float2 y) {
  y.x = max_nan(y.x, -125.0f);
  y.y = max_nan(y.y, -125.0f);
  const float2 t = __fadd2_rn(y, make_float2(12582912.0f, 12582912.0f));
  const float2 r = __fadd2_rn(t, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = __ffma2_rn(r, make_float2(-1.0f, -1.0f), y);
  float2 p = make_float2(0.0013276450335979462f, 0.0013276450335979462f);
  p = __ffma2_rn(p, f, make_float2(0.00967553909868002f, 0.00967553909868002f));
  p = __ffma2_rn(p, f, make_float2(0.05550713464617729f, 0.05550713464617729f));
  p = __ffma2_rn(p, f, make_float2(0.24022120237350464f, 0.24022120237350464f));
  p = __ffma2_rn(p, f, make_float2(0.6931469440460205f, 0.6931469440460205f));
  p = __ffma2_rn(p, f, make_float2(1.0000001192092896f, 1.0000001192092896f));
  // 2^r: r << 23 (the low bits of t shifted into the exponent field) + the bias
  const float2 s2 = make_float2(__int_as_float((__float_as_int(t.x) << 23) + (127 << 23)),
                                __int_as_float((__float_as_int(t.y) << 23) + (127 << 23)));
  return __fmul2_rn(p, s2);
}

// Of a thread's 8 chunks of a piece, this many take their pass-1 exponentials
// from exp2_fma2 (the rest from ex2.approx on the MUFU pipe): for long rows,
// whose pass 1 runs on its own, moving a quarter of them measured 2.8% faster;
// for the short rows' interleaved passes it measured 4% slower.
#ifndef GH_RING_FMA_EXP_LONG
#define GH_RING_FMA_EXP_LONG 2
#endif
#ifndef GH_RING_FMA_EXP_SHORT
#define GH_RING_FMA_EXP_SHORT 0
#endif
constexpr int kFmaExpChunksLong = GH_RING_FMA_EXP_LONG;
constexpr int kFmaExpChunksShort = GH_RING_FMA_EXP_SHORT;

// One thread's share of a full piece: chunks gtid + i * kGroupThreads
// (i < 8), already in registers.  One max test and at most one rescale cover
// all eight, and the exponentials go to four independent accumulators.
template <typename T, int EMU = 0>
__device__ __forceinline__ void fold_full_piece(MaxSum& st, const uint4 (&q)[kPieceChunksPerThread]) {
  constexpr int EPC = 16 / Elem<T>::kBytes;
  constexpr int K = kPieceChunksPerThread;
  float cm;
  if constexpr (EPC == 8) {
    uint32_t m4[4] = {q[0].x, q[0].y, q[0].z, q[0].w};
#pragma unroll
    for (int i = 1; i < K; ++i) {
      m4[0] = bf16x2_max(m4[0], q[i].x);
      m4[1] = bf16x2_max(m4[1], q[i].y);
      m4[2] = bf16x2_max(m4[2], q[i].z);
      m4[3] = bf16x2_max(m4[3], q[i].w);
    }
    const uint32_t mx = bf16x2_max(bf16x2_max(m4[0], m4[1]), bf16x2_max(m4[2], m4[3]));
    cm = fmaxf(bf16_lo(mx), bf16_hi(mx));
  } else {
    float m4[4] = {__uint_as_float(q[0].x), __uint_as_float(q[0].y), __uint_as_float(q[0].z),
                   __uint_as_float(q[0].w)};
#pragma unroll
    for (int i = 1; i < K; ++i) {
      m4[0] = fmaxf(m4[0], __uint_as_float(q[i].x));
      m4[1] = fmaxf(m4[1], __uint_as_float(q[i].y));
      m4[2] = fmaxf(m4[2], __uint_as_float(q[i].z));
      m4[3] = fmaxf(m4[3], __uint_as_float(q[i].w));
    }
    cm = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
  }
  raise_ref(st, cm);
  if (st.m == kNegInf) return;  // only -inf logits so far
  const float nm = -st.m * kLog2e;
  const float2 l2 = make_float2(kLog2e, kLog2e), nm2 = make_float2(nm, nm);
  float2 acc[4] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f),
                   make_float2(0.0f, 0.0f)};
#pragma unroll
  for (int i = 0; i < K; ++i) {
    float v[EPC];
    unpack16<T>(q[i], v);
#pragma unroll
    for (int j = 0; j < EPC; j += 2) {
      const float2 y = __ffma2_rn(make_float2(v[j], v[j + 1]), l2, nm2);
      float2& ac = acc[(i * EPC / 2 + j / 2) & 3];
      ac = __fadd2_rn(ac, i < EMU ? exp2_fma2(y) : make_float2(ex2(y.x), ex2(y.y)));
    }
  }
  const float2 a01 = __fadd2_rn(acc[0], acc[1]), a23 = __fadd2_rn(acc[2], acc[3]);
  const float2 a = __fadd2_rn(a01, a23);
  st.s += a.x + a.y;
}

// One chunk of a short piece (a row's last), folded on its own.
template <typename T>
__device__ __forceinline__ void fold_one(MaxSum& st, const uint4& q) {
  constexpr int EPC = 16 / Elem<T>::kBytes;
  float v[EPC];
  unpack16<T>(q, v);
  float cm = v[0];
#pragma unroll
  for (int i = 1; i < EPC; ++i) cm = fmaxf(cm, v[i]);
  raise_ref(st, cm);
  if (st.m == kNegInf) return;
  const float nm = -st.m * kLog2e;
  float acc = 0.0f;
#pragma unroll
  for (int i = 0; i < EPC; ++i) acc += ex2(fmaf(v[i], kLog2e, nm));
  st.s += acc;
}

template <typename T, int MODE>
__global__ void __launch_bounds__(kRingThreads, 1) ce_ring_kernel(CeArgs a) {
  constexpr int ES = Elem<T>::kBytes;
  extern __shared__ __align__(128) uint8_t smem[];
  RingShared& sh = *reinterpret_cast<RingShared*>(smem);
  uint8_t* ring = smem + kRingHdrBytes;
  const int warp = static_cast<int>(threadIdx.x) >> 5, lane = static_cast<int>(threadIdx.x) & 31;
  const int64_t G = gridDim.x;
  const int64_t first = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kRingSlots; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], kGroupWarps);
    }
    for (int i = 0; i < kRingFinalizers; ++i) {
      mbar_init(&sh.rowfull[i], kRingConsumerWarps);
      mbar_init(&sh.rowempty[i], 1);
    }
    sh.abort = 0;
    fence_mbar_init();
  }
  pdl_wait();     // the predecessor's outputs (targets, logits) are complete
  pdl_trigger();  // persistent grid: the next kernel may start launching
  __syncthreads();

  volatile int* abort_flag = &sh.abort;
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity)) return true;
    *abort_flag = 1;
    return false;
  };
  auto target_of = [&](int64_t row) -> int64_t { return row < a.B ? a.targets[row] : int64_t(0); };

  if (warp == kRingConsumerWarps) {
    // ---------------- producer ----------------
    if (lane == 0) {
      uint32_t n = 0;  // pieces issued
      int64_t t = target_of(first);
      for (int64_t row = first; row < a.B; row += G) {
        const int64_t t_next = target_of(row + G);
        if (ring_target_valid(a, t)) {
          const RingRow r = ring_row<ES>(a, row);
          const int np = ring_pieces(r);
          for (int p = 0; p < np; ++p, ++n) {
            const int s = static_cast<int>(n % kRingSlots);
            if (!wait(&sh.empty[s], ((n / kRingSlots) & 1) ^ 1)) break;
            const int c0 = r.c_lo + p * kRingPieceChunks;
            const uint32_t bytes = 16u * static_cast<uint32_t>(tmin(kRingPieceChunks, r.c_hi - c0));
            mbar_arrive_expect_tx(&sh.full[s], bytes);
            bulk_g2s(ring + s * kRingPieceBytes, r.base + 16 * static_cast<int64_t>(c0), bytes, &sh.full[s]);
          }
        }
        if (*abort_flag) break;
        t = t_next;
      }
      // On an abort, the copies still in flight land before the CTA exits.
      if (*abort_flag) {
        for (uint32_t k = (n > kRingSlots ? n - kRingSlots : 0); k < n; ++k)
          (void)mbar_wait(&sh.full[k % kRingSlots], (k / kRingSlots) & 1);
      }
    }
    return;
  }

  if (warp > kRingConsumerWarps) {
    // ---------------- finalizers ----------------
    const uint32_t f = warp - kRingConsumerWarps - 1;
    uint32_t k = 0;  // valid rows seen
    uint32_t i = 0;  // rows seen
    int64_t t = target_of(first);
    for (int64_t row = first; row < a.B; row += G, ++i) {
      const int64_t t_next = target_of(row + G);
      if (!ring_target_valid(a, t)) {
        if (lane == 0 && i % kRingFinalizers == f) {
          if constexpr (MODE == kModeSelect) {
            a.row_loss[row] = __int_as_float(0x7fc00000);
            record_status(GH_ERR_TARGET_RANGE);
          } else {
            a.row_loss[row] = 0.0f;
          }
        }
        t = t_next;
        continue;
      }
      if (k % kRingFinalizers != f) {
        ++k;
        t = t_next;
        continue;
      }
      const RingRow r = ring_row<ES>(a, row);
      const uint8_t* src = static_cast<const uint8_t*>(a.logits) + row * a.ld * ES;
      // ragged ends: lanes 0-15 the head elements, lanes 16-31 the tail
      float edge = kNegInf;
      if (lane < 16) {
        if (lane < r.h) edge = Elem<T>::load(src + static_cast<int64_t>(lane) * ES);
      } else {
        const int64_t e = r.tail + (lane - 16);
        if (e < a.V) edge = Elem<T>::load(src + e * ES);
      }
      const float xt = Elem<T>::load(src + t * ES);
      const int j = static_cast<int>(f);
      const bool ok = __all_sync(0xffffffffu, wait(&sh.rowfull[j], (k / kRingFinalizers) & 1));
      MaxSum st = ok ? merge_lane_states(sh.part[j], lane) : MaxSum{kNegInf, 0.0f};
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.rowempty[j]);
      st = combine(st, edge == kNegInf ? MaxSum{kNegInf, 0.0f} : MaxSum{edge, 1.0f});
      st = warp_reduce(st);
      if (lane == 0) {
        const float lse = st.m + logf(st.s);
        a.row_loss[row] = MODE == kModeSelect ? xt - lse : (lse - xt) + a.z * lse * lse;
      }
      ++k;
      t = t_next;
      if (!ok) break;
    }
    return;
  }

  // ---------------- consumers ----------------
  // Each thread posts its own (max, sum) state of valid row k for the row's
  // finalizer (no reduction here: the finalizer merges the 512 states).
  auto post_state = [&](const MaxSum& st, uint32_t k) {
    const int j = static_cast<int>(k % kRingFinalizers);
    bool free_slot = true;
    if (lane == 0) free_slot = wait(&sh.rowempty[j], ((k / kRingFinalizers) & 1) ^ 1);
    __syncwarp();
    if (__shfl_sync(0xffffffffu, free_slot ? 1 : 0, 0)) {
      sh.part[j][warp][lane] = make_float2(st.m, st.s);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.rowfull[j]);
    }
    __syncwarp();
  };
  const int grp = warp / kGroupWarps;
  const int gtid = static_cast<int>(threadIdx.x) - grp * kGroupThreads;
  uint32_t n = 0;  // pieces seen (this group consumes n % kRingGroups == grp)
  uint32_t k = 0;  // valid rows
  int64_t t = target_of(first);
  for (int64_t row = first; row < a.B; row += G) {
    const int64_t t_next = target_of(row + G);
    if (!ring_target_valid(a, t)) {
      t = t_next;
      continue;
    }
    const RingRow r = ring_row<ES>(a, row);
    const int np = ring_pieces(r);
    const int nbc = r.c_hi - r.c_lo;
    MaxSum st{kNegInf, 0.0f};
    bool ok = true;
    for (int p = 0; p < np; ++p, ++n) {
      if (static_cast<int>(n % kRingGroups) != grp) continue;
      const int s = static_cast<int>(n % kRingSlots);
      if (!__all_sync(0xffffffffu, wait(&sh.full[s], (n / kRingSlots) & 1))) {
        ok = false;
        break;
      }
      const uint8_t* piece = ring + s * kRingPieceBytes;
      const int nc = tmin(kRingPieceChunks, nbc - p * kRingPieceChunks);
      if (nc == kRingPieceChunks) {
        // a full piece: into registers, the slot back to the producer (the
        // arrive's release orders it after the loads), then the arithmetic
        uint4 q[kPieceChunksPerThread];
#pragma unroll
        for (int i = 0; i < kPieceChunksPerThread; ++i)
          q[i] = *reinterpret_cast<const uint4*>(piece + 16 * (gtid + i * kGroupThreads));
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[s]);
        fold_full_piece<T>(st, q);
      } else {
        for (int c = gtid; c < nc; c += kGroupThreads) fold_one<T>(st, *reinterpret_cast<const uint4*>(piece + 16 * c));
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[s]);
      }
    }
    if (!ok) break;
    post_state(st, k);
    if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
    ++k;
    t = t_next;
  }
}


// ---------------------------------------------------------------------------
// Forward and backward: two passes over every row through the same ring.
//
// Pass 1 of row k is the forward kernel's (online max / sum, the finalizer
// merges, writes the row loss and publishes lse); pass 2 of row k copies the
// row into the ring again and stores the gradient scale (1 + 2 z lse) exp(x -
// lse), less scale at the target, straight from registers to global.  For
// rows shorter than kLongRowBytes the producer interleaves the passes one row
// apart -- pass 1 of row k, then pass 2 of row k - 1 -- so lse(k - 1) is ready
// when its pass 2 lands and the row was read from HBM one row earlier: the
// second copy comes from L2.  Longer rows run pass 2 straight after their own
// pass 1, with L2 eviction hints (below).  HBM sees one read and one write of
// every logit; every element costs two exponentials.  Ignored rows skip both
// copies and get a zero gradient row.
// ---------------------------------------------------------------------------

// Pass 2 of a row follows pass 1 of the next row, so lse is ready when its
// copies land and the consumers never wait on the finalizer.  For rows of
// kLongRowBytes or more that order puts about three rows of other traffic
// between the two copies of a piece (3 x 148 x 128 KiB = 57 MB and up, 227 MB
// for 512 KiB rows: too much for L2 next to the gradient stores), so pass 2
// would read HBM again (measured: 112 KiB rows run at 82% of the copy rate
// in this order, 128 KiB rows at 72%); those rows
// run pass 2 straight after their own pass 1 instead (about one row between
// the copies), and the consumers wait for the row's lse once, while the
// producer's pass-2 copies are already in flight.  Their pass-1 copies mark
// the lines evict-last and the pass-2 copies evict-first, so the row stays in
// L2 between the two (the gradient stores are evict-first too), and pass 2
// walks the row backwards: the pieces pass 1 read last are re-read first.
#ifndef GH_RING_LONG_ROW_BYTES
#define GH_RING_LONG_ROW_BYTES (120 * 1024)
#endif
constexpr int64_t kLongRowBytes = GH_RING_LONG_ROW_BYTES;

// Gradient of one 16-byte chunk: element e0 + j of the row gets
// coef 2^(x_j log2e + nl) (nl = -lse log2e), minus scale at the target (chunk
// position tj, or -1).  `dst` is the chunk's first element in the gradient row.
template <typename T>
__device__ __forceinline__ void grad_chunk(const uint4& q, float coef, float nl, int tj, float scale, uint8_t* dst,
                                           bool congruent) {
  constexpr int EPC = 16 / Elem<T>::kBytes;
  constexpr int ES = Elem<T>::kBytes;
  float v[EPC], g[EPC];
  unpack16<T>(q, v);
  const float2 l2 = make_float2(kLog2e, kLog2e), nl2 = make_float2(nl, nl), c2 = make_float2(coef, coef);
#pragma unroll
  for (int j = 0; j < EPC; j += 2) {
    const float2 y = __ffma2_rn(make_float2(v[j], v[j + 1]), l2, nl2);
    const float2 r = __fmul2_rn(make_float2(ex2(y.x), ex2(y.y)), c2);
    g[j] = r.x;
    g[j + 1] = r.y;
  }
  if (tj >= 0) {
#pragma unroll
    for (int j = 0; j < EPC; ++j)
      if (j == tj) g[j] -= scale;
  }
  if (congruent) {
    __stcs(reinterpret_cast<uint4*>(dst), pack16<T>(g));
  } else {
#pragma unroll
    for (int j = 0; j < EPC; ++j) Elem<T>::store(dst + j * ES, g[j]);
  }
}

// LONG: rows of kLongRowBytes or more (pass 2 right after the row's own pass 1,
// cache-hinted copies).  The order is a template parameter so that each
// instantiation inlines the two passes once (the instruction cache is small).
template <typename T, bool LONG>
__global__ void __launch_bounds__(kRingThreads, 1) ce_ring2_kernel(CeArgs a) {
  constexpr int ES = Elem<T>::kBytes;
  constexpr bool lag0 = LONG;
  extern __shared__ __align__(128) uint8_t smem[];
  RingShared& sh = *reinterpret_cast<RingShared*>(smem);
  uint8_t* ring = smem + kRingHdrBytes;
  const int warp = static_cast<int>(threadIdx.x) >> 5, lane = static_cast<int>(threadIdx.x) & 31;
  const int64_t G = gridDim.x;
  const int64_t first = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kRingSlots; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], kGroupWarps);
    }
    for (int i = 0; i < kRingFinalizers; ++i) {
      mbar_init(&sh.rowfull[i], kRingConsumerWarps);
      mbar_init(&sh.rowempty[i], 1);
      mbar_init(&sh.lseready[i], 1);
    }
    sh.abort = 0;
    fence_mbar_init();
  }
  pdl_wait();     // the predecessor's outputs (targets, logits, n_valid) are complete
  pdl_trigger();  // persistent grid: the next kernel may start launching
  __syncthreads();

  volatile int* abort_flag = &sh.abort;
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity)) return true;
    *abort_flag = 1;
    return false;
  };
  auto target_of = [&](int64_t row) -> int64_t { return row < a.B ? a.targets[row] : int64_t(0); };
  auto grad_row = [&](int64_t row) -> uint8_t* { return static_cast<uint8_t*>(a.grad) + row * a.ld * ES; };
  // byte phase of a logits row within its 16-byte chunk
  auto row_lead = [&](int64_t row) -> int {
    return static_cast<int>((reinterpret_cast<uintptr_t>(a.logits) + static_cast<uintptr_t>(row * a.ld * ES)) & 15);
  };

  if (warp == kRingConsumerWarps) {
    // ---------------- producer: pass 1 of row i, then pass 2 of row i - 1 ----------------
    if (lane == 0) {
      uint32_t n = 0;  // pieces issued
      // long rows: pass-1 copies keep their lines in L2 for pass 2, pass-2
      // copies let them go
      const uint64_t pol_keep = l2_policy_evict_last(), pol_drop = l2_policy_evict_first();
      auto issue_row = [&](int64_t row, bool first_pass) -> bool {
        const RingRow r = ring_row<ES>(a, row);
        const int np = ring_pieces(r);
        for (int q = 0; q < np; ++q, ++n) {
          const int p = (lag0 && !first_pass) ? np - 1 - q : q;  // long rows: pass 2 backwards
          const int s = static_cast<int>(n % kRingSlots);
          if (!wait(&sh.empty[s], ((n / kRingSlots) & 1) ^ 1)) return false;
          if (a.withhold_plus1 != 0 && blockIdx.x == 0 && n + 1 == a.withhold_plus1) continue;  // test of the failure path
          const int c0 = r.c_lo + p * kRingPieceChunks;
          const uint32_t bytes = 16u * static_cast<uint32_t>(tmin(kRingPieceChunks, r.c_hi - c0));
          mbar_arrive_expect_tx(&sh.full[s], bytes);
          if constexpr (lag0)
            bulk_g2s_hint(ring + s * kRingPieceBytes, r.base + 16 * static_cast<int64_t>(c0), bytes, &sh.full[s],
                          first_pass ? pol_keep : pol_drop);
          else
            bulk_g2s(ring + s * kRingPieceBytes, r.base + 16 * static_cast<int64_t>(c0), bytes, &sh.full[s]);
        }
        return true;
      };
      int64_t t = target_of(first);
      bool prev_valid = false;
      for (int64_t row = first;; row += G) {
        const bool has = row < a.B;
        const int64_t t_next = has ? target_of(row + G) : 0;
        const bool valid = has && ring_target_valid(a, t);
        if (valid && !issue_row(row, true)) break;
        if constexpr (lag0) {
          if (valid && !issue_row(row, false)) break;
        } else if (prev_valid && !issue_row(row - G, false)) {
          break;
        }
        if (!has || *abort_flag) break;
        prev_valid = valid;
        t = t_next;
      }
      if (*abort_flag) {  // the copies still in flight land before the CTA exits
        for (uint32_t k = (n > kRingSlots ? n - kRingSlots : 0); k < n; ++k)
          (void)mbar_wait(&sh.full[k % kRingSlots], (k / kRingSlots) & 1);
      }
    }
    return;
  }

  const unsigned long long nv = *a.n_valid;
  const float scale = a.mean ? 1.0f / static_cast<float>(nv > 0 ? nv : 1ull) : 1.0f;

  if (warp > kRingConsumerWarps) {
    // ---------------- finalizers ----------------
    const uint32_t f = warp - kRingConsumerWarps - 1;
    uint32_t k = 0;  // valid rows seen
    uint32_t i = 0;  // rows seen
    int64_t t = target_of(first);
    for (int64_t row = first; row < a.B; row += G, ++i) {
      const int64_t t_next = target_of(row + G);
      if (!ring_target_valid(a, t)) {
        if (lane == 0 && i % kRingFinalizers == f) a.row_loss[row] = 0.0f;
        t = t_next;
        continue;
      }
      if (k % kRingFinalizers != f) {
        ++k;
        t = t_next;
        continue;
      }
      const RingRow r = ring_row<ES>(a, row);
      const uint8_t* src = static_cast<const uint8_t*>(a.logits) + row * a.ld * ES;
      // ragged ends: lanes 0-15 the head elements, lanes 16-31 the tail
      int64_t e = -1;
      if (lane < 16) {
        if (lane < r.h) e = lane;
      } else if (r.tail + (lane - 16) < a.V) {
        e = r.tail + (lane - 16);
      }
      const float edge = e >= 0 ? Elem<T>::load(src + e * ES) : kNegInf;
      const float xt = Elem<T>::load(src + t * ES);
      const int j = static_cast<int>(f);
      const bool ok = __all_sync(0xffffffffu, wait(&sh.rowfull[j], (k / kRingFinalizers) & 1));
      MaxSum st = ok ? merge_lane_states(sh.part[j], lane) : MaxSum{kNegInf, 0.0f};
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.rowempty[j]);
      st = combine(st, edge == kNegInf ? MaxSum{kNegInf, 0.0f} : MaxSum{edge, 1.0f});
      st = warp_reduce(st);
      const float lse = st.m + logf(st.s);
      if (lane == 0) {
        sh.lse[j] = lse;
        mbar_arrive(&sh.lseready[j]);
        a.row_loss[row] = (lse - xt) + a.z * lse * lse;
      }
      if (e >= 0) {  // the ragged ends' gradient
        const float coef = scale * (1.0f + 2.0f * a.z * lse);
        float g = coef * ex2(fmaf(edge, kLog2e, -lse * kLog2e));
        if (e == t) g -= scale;
        Elem<T>::store(grad_row(row) + e * ES, g);
      }
      ++k;
      t = t_next;
      if (!ok) break;
    }
    return;
  }

  // ---------------- consumers ----------------
  // Each thread posts its own (max, sum) state of valid row k for the row's
  // finalizer (no reduction here: the finalizer merges the 512 states).
  auto post_state = [&](const MaxSum& st, uint32_t k) {
    const int j = static_cast<int>(k % kRingFinalizers);
    bool free_slot = true;
    if (lane == 0) free_slot = wait(&sh.rowempty[j], ((k / kRingFinalizers) & 1) ^ 1);
    __syncwarp();
    if (__shfl_sync(0xffffffffu, free_slot ? 1 : 0, 0)) {
      sh.part[j][warp][lane] = make_float2(st.m, st.s);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.rowfull[j]);
    }
    __syncwarp();
  };
  const int grp = warp / kGroupWarps;
  const int gtid = static_cast<int>(threadIdx.x) - grp * kGroupThreads;
  const int tid = static_cast<int>(threadIdx.x);
  uint32_t n = 0;  // pieces seen (this group consumes n % kRingGroups == grp)
  uint32_t k = 0;  // valid rows seen
  bool ok = true;

  // pass 1 of a valid row: the online (max, sum) state, posted for the finalizer
  auto pass1 = [&](int64_t row) {
    const RingRow r = ring_row<ES>(a, row);
    const int np = ring_pieces(r);
    const int nbc = r.c_hi - r.c_lo;
    MaxSum st{kNegInf, 0.0f};
    for (int p = 0; p < np; ++p, ++n) {
      if (static_cast<int>(n % kRingGroups) != grp) continue;
      const int s = static_cast<int>(n % kRingSlots);
      if (!__all_sync(0xffffffffu, wait(&sh.full[s], (n / kRingSlots) & 1))) {
        ok = false;
        return;
      }
      const uint8_t* piece = ring + s * kRingPieceBytes;
      const int nc = tmin(kRingPieceChunks, nbc - p * kRingPieceChunks);
      if (nc == kRingPieceChunks) {
        uint4 q[kPieceChunksPerThread];
#pragma unroll
        for (int i = 0; i < kPieceChunksPerThread; ++i)
          q[i] = *reinterpret_cast<const uint4*>(piece + 16 * (gtid + i * kGroupThreads));
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[s]);
        fold_full_piece<T, lag0 ? kFmaExpChunksLong : kFmaExpChunksShort>(st, q);
      } else {
        for (int c = gtid; c < nc; c += kGroupThreads) fold_one<T>(st, *reinterpret_cast<const uint4*>(piece + 16 * c));
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[s]);
      }
    }
    post_state(st, k);
    if (__any_sync(0xffffffffu, *abort_flag != 0)) ok = false;
  };

  // pass 2 of valid row `row` (valid-row index kr, target t): the gradient of
  // its whole chunks
  auto pass2 = [&](int64_t row, int64_t t, uint32_t kr) {
    const RingRow r = ring_row<ES>(a, row);
    const int np = ring_pieces(r);
    const int nbc = r.c_hi - r.c_lo;
    const int j = static_cast<int>(kr % kRingFinalizers);
    // every consumer warp waits for every row's lse, so each lseready phase is
    // observed in order
    if (!__all_sync(0xffffffffu, wait(&sh.lseready[j], (kr / kRingFinalizers) & 1))) {
      ok = false;
      return;
    }
    const float lse = sh.lse[j];
    const float coef = scale * (1.0f + 2.0f * a.z * lse);
    const float nl = -lse * kLog2e;
    const int lead = row_lead(row);
    uint8_t* gbase = grad_row(row) - lead;  // chunk c's gradient bytes start at gbase + 16 c
    const bool congruent = a.congruent != 0;
    const int64_t tb = lead + t * ES;        // target's byte in the row's chunk space
    const int tc = static_cast<int>(tb >> 4), tj = static_cast<int>((tb & 15) / ES);
    for (int q = 0; q < np; ++q, ++n) {
      if (static_cast<int>(n % kRingGroups) != grp) continue;
      const int p = lag0 ? np - 1 - q : q;  // long rows: pass 2 backwards (the producer's order)
      const int s = static_cast<int>(n % kRingSlots);
      if (!__all_sync(0xffffffffu, wait(&sh.full[s], (n / kRingSlots) & 1))) {
        ok = false;
        return;
      }
      const uint8_t* piece = ring + s * kRingPieceBytes;
      const int c0 = r.c_lo + p * kRingPieceChunks;
      const int nc = tmin(kRingPieceChunks, nbc - p * kRingPieceChunks);
      if (nc == kRingPieceChunks) {
        uint4 q[kPieceChunksPerThread];
#pragma unroll
        for (int i = 0; i < kPieceChunksPerThread; ++i)
          q[i] = *reinterpret_cast<const uint4*>(piece + 16 * (gtid + i * kGroupThreads));
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[s]);
#pragma unroll
        for (int i = 0; i < kPieceChunksPerThread; ++i) {
          const int c = c0 + gtid + i * kGroupThreads;
          grad_chunk<T>(q[i], coef, nl, c == tc ? tj : -1, scale, gbase + 16 * static_cast<int64_t>(c), congruent);
        }
      } else {
        for (int cc = gtid; cc < nc; cc += kGroupThreads) {
          const int c = c0 + cc;
          grad_chunk<T>(*reinterpret_cast<const uint4*>(piece + 16 * cc), coef, nl, c == tc ? tj : -1, scale,
                        gbase + 16 * static_cast<int64_t>(c), congruent);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[s]);
      }
    }
  };

  // an ignored row: zero gradient (whole chunks and ragged ends), no copies
  auto zero_row = [&](int64_t row) {
    const RingRow r = ring_row<ES>(a, row);
    uint8_t* g = grad_row(row);
    uint8_t* gbase = g - row_lead(row);
    if (a.congruent) {
      for (int c = r.c_lo + tid; c < r.c_hi; c += kRingConsumers)
        __stcs(reinterpret_cast<uint4*>(gbase + 16 * static_cast<int64_t>(c)), make_uint4(0, 0, 0, 0));
    } else {
      for (int64_t e = r.h + tid; e < r.tail; e += kRingConsumers) Elem<T>::store(g + e * ES, 0.0f);
    }
    if (tid < r.h) Elem<T>::store(g + static_cast<int64_t>(tid) * ES, 0.0f);
    if (tid >= 32 && tid < 48 && r.tail + (tid - 32) < a.V) Elem<T>::store(g + (r.tail + (tid - 32)) * ES, 0.0f);
  };

  int64_t t = target_of(first);
  bool prev_valid = false;
  int64_t prev_t = 0;
  uint32_t prev_k = 0;
  for (int64_t row = first;; row += G) {
    const bool has = row < a.B;
    const int64_t t_next = has ? target_of(row + G) : 0;
    const bool valid = has && ring_target_valid(a, t);
    const uint32_t kr = k;
    if (valid) {
      pass1(row);
      ++k;
      if (!ok) break;
    }
    if constexpr (lag0) {  // pass 2 (or the zero row) of this row
      if (valid) {
        pass2(row, t, kr);
        if (!ok) break;
      } else if (has) {
        zero_row(row);
      }
    } else if (row - G >= first) {  // pass 2 (or the zero row) of the previous row
      if (prev_valid) {
        pass2(row - G, prev_t, prev_k);
        if (!ok) break;
      } else {
        zero_row(row - G);
      }
    }
    if (!has) break;
    prev_valid = valid;
    prev_t = t;
    prev_k = kr;
    t = t_next;
  }
}

// 2^y for n values, by either route the kernels take: method 0 ex2.approx (the
// MUFU pipe), method 1 exp2_fma2 (the FMA pipe, y <= 0).  Diagnostic only.
__global__ void exp2_eval_kernel(const float* __restrict__ y, float* __restrict__ out, int64_t n, int method) {
  const int64_t i = 2 * (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float y0 = y[i], y1 = i + 1 < n ? y[i + 1] : 0.0f;
  const float2 r = method == 1 ? exp2_fma2(make_float2(y0, y1)) : make_float2(ex2(y0), ex2(y1));
  out[i] = r.x;
  if (i + 1 < n) out[i + 1] = r.y;
}

using RingKernel = void (*)(CeArgs);

template <typename T>
RingKernel ring_kernel_mode(int mode) {
  return mode == kModeSelect ? ce_ring_kernel<T, kModeSelect> : ce_ring_kernel<T, kModeFwd>;
}

RingKernel ring_kernel_for(int es, int mode) {
  return es == 4 ? ring_kernel_mode<float>(mode) : ring_kernel_mode<uint16_t>(mode);
}

}  // namespace

int ce_ring_smem_bytes() { return kRingHdrBytes + kRingSlots * kRingPieceBytes; }

gh_status_t exp2_eval_launch(const float* y, float* out, int64_t n, int method, cudaStream_t stream) {
  if (n == 0) return GH_OK;
  constexpr int kThreads = 256;
  const int64_t blocks = ((n + 1) / 2 + kThreads - 1) / kThreads;
  note_launch();
  exp2_eval_kernel<<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(y, out, n, method);
  return cudaGetLastError() == cudaSuccess ? GH_OK : GH_ERR_CUDA;
}

gh_status_t ce_ring_launch(const CeArgs& args, int es, int grid, cudaStream_t stream) {
  CeArgs a = args;
  const bool long_rows = a.V * es >= kLongRowBytes;
  RingKernel kern;
  if (a.mode == kModeFwdBwd) {
    a.withhold_plus1 = debug_ring_piece().exchange(-1) + 1;
    if (es == 4) kern = long_rows ? ce_ring2_kernel<float, true> : ce_ring2_kernel<float, false>;
    else kern = long_rows ? ce_ring2_kernel<uint16_t, true> : ce_ring2_kernel<uint16_t, false>;
  } else {
    kern = ring_kernel_for(es, a.mode);
  }
  if (ensure_smem_limit(kern, ce_ring_smem_bytes()) != cudaSuccess) return GH_ERR_CUDA;
  ProfileScope prof(a.profile_kind, stream);
  note_launch();
  return launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(kRingThreads), ce_ring_smem_bytes(), stream, 1,
                    a) == cudaSuccess
             ? GH_OK
             : GH_ERR_CUDA;
}

}  // namespace gh
