// Persistent bf16 GEMM on the sm_100a tensor cores (tcgen05.mma, TMEM
// accumulators, TMA operand loads), written for the three contractions of the
// chunked linear cross-entropy (Greyhound `chunked_linear_loss`):
//
//   logits_c = X_c  W^T   A = X_c [rows, D]   K-major    B = W   [V, D]    K-major
//   dX_c     = G_c  W     A = G_c [rows, V]   K-major    B = W   [V, D]    N-major
//   dW      += G_c^T X_c  A = G_c^T           M-major    B = X_c [rows, D] N-major
//
// For the cross-entropy the logits tile never leaves the chip as logits: the
// epilogue (kEpiCeExp) turns each fp32 value into exp(x - R_row) and keeps the
// row's sum and max over the tile, so the gradient GEMMs take G = diag(alpha) P
// with P the stored exponentials (the row factor alpha is applied in the dX
// epilogue as a row scale, and folded into X_c for dW).
//
// D[M, N] = sum_k A[m, k] B[n, k], in 64-wide K steps, on tiles of 128 x 256
// computed by one CTA (cta_group::1) or of 256 x 256 computed by a pair of CTAs
// in a cluster (cta_group::2: each CTA loads its 128 A rows and 128 of the 256
// B rows, the leader issues the MMAs, each CTA's TMEM holds its 128 rows).
// Warp roles in each CTA:
//   warps 0, 6  TMA producers (one lane each, alternate stages): A and B
//               tiles into a ring of shared-memory stages, 128-byte swizzled;
//               a pair's stage barrier lives in the leader and counts both
//               CTAs' bytes.  G_c (the chunk's exponentials) is stored in
//               64-column blocks and read through 3-D maps, so each A tile of
//               dX and dW is one contiguous piece of memory
//   warp 1      TMEM allocator; in the leader, the MMA issuer (one lane):
//               4 x tcgen05.mma (K=16) per stage, commits release the stage
//               (in both CTAs) and publish finished accumulators
//   warps 2..5  epilogue: tcgen05.ld of the fp32 accumulator (each warp owns
//               the 32 TMEM lanes its warp id selects), conversion, and TMA
//               stores, reduce-adds or read-add-store of the output through
//               two staging buffers per warp
// Two accumulators of 256 fp32 columns (all 512 TMEM columns) let the
// epilogue of one tile overlap the MMAs of the next.  Every wait is bounded
// (GH_ERR_TIMEOUT, then all roles stop, copies in flight land, the MMAs
// finish and TMEM is freed).  No load is multicast.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace gh {
namespace sm100 {

constexpr int kBM = 128;                      // accumulator rows of one CTA (TMEM lanes)
constexpr int kBN = 256;                      // accumulator columns (one tcgen05.mma N)
constexpr int kBK = 64;                       // one 128-byte swizzle row of bf16
constexpr int kABytes = kBM * kBK * 2;        // 16 KiB
constexpr int kGemmThreads = 224;  // producer, MMA, 4 epilogue warps, second producer
constexpr int kTmemCols = 2 * kBN;            // two accumulators
constexpr int kStageOutBytes = 4096;          // one epilogue staging buffer: 32 rows x 128 bytes
constexpr int kOutBytes = 4 * 2 * kStageOutBytes;  // 4 epilogue warps x 2 buffers

// One CTA per tile (cta_group::1: 128 x 256 tiles, the CTA loads all 256 B
// rows) or a CTA pair per tile (cta_group::2: 256 x 256 tiles, each CTA loads
// its 128 A rows and 128 of the B rows, the leader issues the MMAs for both).
// With half the B bytes per stage, the pair keeps 6 stages in flight where a
// single CTA keeps 4, in the same shared memory.
template <bool PAIR>
struct GemmCfg {
  static constexpr int kTileM = PAIR ? 2 * kBM : kBM;  // output rows of a tile
  static constexpr int kBRows = PAIR ? kBN / 2 : kBN;  // B rows (N) this CTA loads per stage
  static constexpr int kStages = PAIR ? 6 : 4;
  static constexpr int kBBytes = kBRows * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kSmem = 1024 /*align*/ + kStages * kStageBytes + kOutBytes + 256 /*barriers*/;
};
constexpr int kGemmSmem = GemmCfg<false>::kSmem;
constexpr int kMaxSplits = 4;  // K splits a tile may be cut into when they are summed in the kernel
constexpr int kProducers = 2;  // TMA producer warps (warps 0 and 6)
static_assert(GemmCfg<true>::kSmem <= 232448 && GemmCfg<false>::kSmem <= 232448, "shared memory per CTA");

// Epilogue modes (what happens to the fp32 tile).  The first three go out
// through the `tma_out` tensor map from a swizzled shared-memory staging
// buffer per epilogue warp; TMA clips rows and columns outside the map.
enum GemmEpi : int {
  kEpiStoreBf16 = 0,  // out(bf16) = tile                       TMA store
  kEpiStoreF32 = 1,   // out(f32)  = tile                       TMA store
  kEpiAddF32 = 2,     // out(f32) += tile                       TMA reduce-add (in L2)
  kEpiBf16Add = 3,    // out(bf16) = bf16(out + tile)          TMA load, add in place, TMA store
  kEpiCeExp = 4,      // logits tile of the fused cross-entropy: out(bf16) = exp(tile - R_row)
                      // (0 for ignored rows), plus per (row, column tile) sum and max
  kEpiAccToBf16 = 5   // out(bf16) = bf16(acc + tile), acc the fp32 array of `tma_aux`   TMA loads and store
};

struct GemmArgs {
  int M, N, K;
  int tiles_m, tiles_n, num_kb;
  int k_splits;         // K is cut into k_splits ranges of kb_per_split K-steps
  int kb_per_split;
  int split_rows;       // row offset in the output map between K splits
  int m_fastest;        // tile order: consecutive tiles share the B tile (1) or the A tile (0)
  int epi;
  // kEpiStoreBf16 / kEpiStoreF32: when non-null, output row r (of the M rows)
  // is multiplied by row_scale[r] before it is stored.
  const float* row_scale;
  // kEpiCeExp: the logits tile of one chunk, M = chunk rows, N = V columns.
  const int64_t* targets;  // [M] class ids; a row whose target is ignore_index or outside [0, N) is stored as 0
  int64_t ignore_index;
  float2* stats;           // [tiles_n][stats_ld]: (sum over the tile's columns of exp(x - R_row), max x)
  int stats_ld;
  float* x_target;         // [M]: the fp32 logit at the row's target column (valid rows)
  const float* row_ref;    // [M] R_row, or null for R_row = 0
  const int* run_flag;     // non-null: the kernel does nothing unless *run_flag != 0
  // kEpiStoreF32 with k_splits > 1 and split_out non-null: the K splits are
  // summed in the kernel.  Each split stores its fp32 partial (rows
  // ks * split_rows + r of split_ws, row stride N); the last split to finish a
  // 32-row slice of a tile adds the slice's partials in split order (the same
  // order whichever split finishes last) and writes bf16 rows of split_out.
  const float* split_ws;
  uint16_t* split_out;
  int64_t split_ld;
  int* split_count;        // one counter per (tile, CTA of the pair, 32-row slice)
  // 0: the last split to finish a slice sums it (counters back to 0 after each
  // launch).  > 0: every unit of the launch is resident at once, and each split
  // waits (bounded) until the slice's counter reaches split_target, then sums
  // every k_splits-th row of the slice (counters only grow within a call).
  int split_target;
  // The chunk's exponentials in the column-blocked layout, through 3-D maps:
  // a_blocked, the A operand (dX: K-major boxes {64, 128, 1}; dW: M-major boxes
  // {64, 64, 2}, both 64-column blocks of a CTA's 128 A columns in one copy);
  // out_blocked, the bf16 output of the epilogue (boxes {64, 32, 2}: two column blocks per copy).
  int a_blocked, out_blocked;
  // failure-path tests: 1 + the stage of unit 0's first tile whose loads the
  // producer leaves out (0: none)
  int withhold_plus1;
  // Start without waiting for the previous kernel on the stream, and wait for
  // it before exiting: for a GEMM that reads nothing the previous kernel
  // writes, when that kernel waited for everything this one reads before it
  // let dependents launch (so this GEMM fills SMs as the previous one's CTAs
  // retire, and still completes after it).
  int defer_wait;
};

// ---- PTX wrappers ----------------------------------------------------------------

__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          smem_u32(smem_dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map),
               "r"(smem_u32(smem_src)), "r"(x), "r"(y)
               : "memory");
}

__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, const void* smem_src, int x, int y) {
  asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   map),
               "r"(smem_u32(smem_src)), "r"(x), "r"(y)
               : "memory");
}

// tma_load_2d into this CTA's shared memory whose completion is counted on an
// mbarrier of either CTA of the pair (`bar` a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(map), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

// 3-D forms for the column-blocked layout of the chunk's exponentials:
// element (row r, column c) at ((c / 64) * block_rows + r) * 64 + c % 64, so a
// box of 64 columns and any run of rows is one contiguous piece of memory.
// Coordinates {c % 64 (always 0 here), r, c / 64}.
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                            int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(smem_u32(smem_dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(void* smem_dst, const CUtensorMap* map, uint32_t bar, int x, int y,
                                                 int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4, %5}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(map), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* smem_src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(map),
               "r"(smem_u32(smem_src)), "r"(x), "r"(y), "r"(z)
               : "memory");
}

// tma_store_3d with an L2 eviction policy (createpolicy).
__device__ __forceinline__ void tma_store_3d_hint(const CUtensorMap* map, const void* smem_src, int x, int y, int z,
                                                  uint64_t policy) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%2, %3, %4}], [%1], %5;" ::"l"(
                   map),
               "r"(smem_u32(smem_src)), "r"(x), "r"(y), "r"(z), "l"(policy)
               : "memory");
}

// Allow at most one committed bulk group still reading shared memory.
__device__ __forceinline__ void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// TMEM allocation: cta_group::2 allocates the same columns in both CTAs of the
// pair, issued by the same warp of each.
template <bool PAIR>
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  if constexpr (PAIR)
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
  else
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
template <bool PAIR>
__device__ __forceinline__ void tmem_relinquish() {
  if constexpr (PAIR)
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  else
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
template <bool PAIR>
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  if constexpr (PAIR)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
  else
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D(tmem) (+)= A(smem desc) x B(smem desc), bf16 inputs, fp32 accumulate.
// cta_group::2: issued by the pair's leader; A rows and B rows come half from
// each CTA's shared memory (same offsets), each CTA's TMEM receives its rows.
template <bool PAIR>
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  if constexpr (PAIR)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once every tcgen05.mma issued so far by this thread is done;
// for a pair, on the barrier at the same offset in both CTAs (a commit, not a
// load: no data moves between the CTAs).
template <bool PAIR>
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  if constexpr (PAIR)
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(static_cast<uint16_t>(3))
        : "memory");
  else
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// tcgen05.wait::ld that also names the registers the loads fill, so no read
// of them can be scheduled before the wait.
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
        "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
        "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
        "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
      :
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&a)[32], uint32_t (&b)[32]) {
  tmem_ld_wait(a);
  tmem_ld_wait(b);  // returns at once: the first wait covered every earlier load
}

// Shared-memory matrix descriptor (tcgen05): start address, leading and
// stride byte offsets (all >> 4), version 1, base offset 0, 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16: bf16 A and B, fp32 D, M x N, majors.
__host__ __device__ constexpr uint32_t instr_desc(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4)            // D format: f32
         | (1u << 7)          // A format: bf16
         | (1u << 10)         // B format: bf16
         | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// One potentially blocking test of phase `parity`, acquiring at cluster scope
// (arrivals may come from the other CTA of a pair).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar_addr, uint32_t parity, uint32_t suspend_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar_addr), "r"(parity), "r"(suspend_ns)
      : "memory");
  return ok != 0;
}

// Wait with an abort flag shared by all roles: returns false once any role
// timed out (and records GH_ERR_TIMEOUT when this wait is the one that did).
template <bool PAIR = false>
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const uint32_t a = smem_u32(bar);
  auto test = [&]() {
    return PAIR ? mbar_try_wait_cluster(a, parity, 20000u) : mbar_try_wait(a, parity, 20000u);
  };
  if (test()) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (test()) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > wait_limit_ns()) {
      *abort_flag = 1;
      record_status(GH_ERR_TIMEOUT);
      return false;
    }
  }
}

// Sleep for about `ns` nanoseconds (bounded by the global timer).
__device__ __forceinline__ void sleep_ns_bounded(uint64_t ns) {
  const uint64_t t0 = global_timer_ns();
  while (global_timer_ns() - t0 < ns) __nanosleep(1000);
}

// ---- the kernel --------------------------------------------------------------------

template <bool A_MN, bool B_MN, bool PAIR = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                     const __grid_constant__ CUtensorMap tma_out, const __grid_constant__ CUtensorMap tma_aux,
                     GemmArgs g) {
  using C = GemmCfg<PAIR>;
  // Each operand layout serves one contraction, so each instantiation keeps
  // only the epilogues that contraction uses (fewer live registers).
  constexpr bool kLogits = !A_MN && !B_MN;  // kEpiCeExp, kEpiStoreBf16
  constexpr bool kDx = !A_MN && B_MN;       // kEpiStoreBf16 (row scale), kEpiStoreF32 (+ split sums)
  constexpr bool kDw = A_MN && B_MN;        // kEpiStoreBf16, kEpiStoreF32, kEpiAddF32, kEpiBf16Add, kEpiAccToBf16
  constexpr int kStages = C::kStages;
  constexpr int kStageBytes = C::kStageBytes;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint8_t* out_stage = smem + kStages * kStageBytes;  // 1024-aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(out_stage + kOutBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tmem_full = empty + kStages;
  uint64_t* tmem_empty = tmem_full + 2;
  uint64_t* mma_done = tmem_empty + 2;
  uint64_t* epi_bar = mma_done + 1;  // kEpiBf16Add: one per epilogue staging buffer
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(epi_bar + 8);
  static_assert((2 * kStages + 2 + 2 + 1 + 8) * 8 + 8 <= 256, "barriers, TMEM address and abort flag");
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // A pair is a cluster of two consecutive CTAs; rank 0 (the leader) issues
  // the MMAs, and its stage and accumulator barriers count both CTAs.
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int unit = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int units = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tmem_full[b], 1);
      mbar_init(&tmem_empty[b], PAIR ? 8 : 4);  // one arrival per epilogue warp (of both CTAs)
    }
    mbar_init(mma_done, 1);
    for (int b = 0; b < 8; ++b) mbar_init(&epi_bar[b], 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tma_a);
    prefetch_tmap(&tma_b);
    prefetch_tmap(&tma_out);
    if (g.epi == kEpiAccToBf16) prefetch_tmap(&tma_aux);
  }
  if (warp == 1) {
    tmem_alloc<PAIR>(tmem_base_slot, kTmemCols);
    tmem_relinquish<PAIR>();
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) {  // both CTAs' barriers are initialised before either signals the other
    cluster_arrive_release();
    cluster_wait_acquire();
  }
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_slot;
  if (!g.defer_wait) pdl_wait();  // operands and outputs are free of the predecessor kernel from here on
  pdl_trigger();  // one CTA per SM, all resident: the next kernel may start its prologue
  // A conditional launch whose flag is clear has no tile to compute (the flag
  // was written by a kernel that completed before pdl_wait returned).
  const int num_tiles_run = (g.run_flag && *reinterpret_cast<const volatile int*>(g.run_flag) == 0)
                                ? 0
                                : g.tiles_m * g.tiles_n * g.k_splits;

  // tile -> (m block, n block, K split); K splits vary slowest
  auto tile_coords = [&](int tile, int& mb, int& nb, int& ks) {
    const int per = g.tiles_m * g.tiles_n;
    ks = tile / per;
    const int t = tile - ks * per;
    if (g.m_fastest) {
      mb = t % g.tiles_m;
      nb = t / g.tiles_m;
    } else {
      nb = t % g.tiles_n;
      mb = t / g.tiles_n;
    }
  };
  auto kb_range = [&](int ks, int& kb0, int& kb1) {
    kb0 = ks * g.kb_per_split;
    kb1 = min(g.num_kb, kb0 + g.kb_per_split);
  };

  if (warp == 0 || warp == 6) {
    // ---------------- TMA producers (both CTAs of a pair: each loads its halves) ----------------
    // Warp 0 and warp 6 each take every other stage load of this CTA's sequence
    // of (tile, K step) items (one issuing thread alone is slower than the loads
    // it issues); kStages is even, so a stage always has the same producer.
    static_assert(kStages % kProducers == 0, "stages per producer");
    if (lane == 0) {
      const int pw = warp == 0 ? 0 : 1;  // this producer's items: pw, pw + kProducers, ...
      int tile = unit, mb = 0, nb = 0, ks = 0, kb0 = 0, kb1 = 0, kb = 0;
      bool have = tile < num_tiles_run;
      if (have) {
        tile_coords(tile, mb, nb, ks);
        kb_range(ks, kb0, kb1);
        kb = kb0;
      }
      auto next_item = [&]() -> bool {  // the next (tile, K step) of this CTA's sequence
        if (++kb < kb1) return true;
        tile += units;
        if (tile >= num_tiles_run) return false;
        tile_coords(tile, mb, nb, ks);
        kb_range(ks, kb0, kb1);
        kb = kb0;
        return kb < kb1;
      };
      for (int i = 0; i < pw && have; ++i) have = next_item();
      uint32_t item = static_cast<uint32_t>(pw);  // linear index of this producer's next load
      uint32_t done = 0;                          // loads this producer issued
      while (have) {
        const int stage = static_cast<int>(item % kStages);
        const uint32_t phase = (item / kStages) & 1u;
        if (!wait_or_abort<PAIR>(&empty[stage], phase ^ 1, abort_flag)) break;
        const bool withhold =
            g.withhold_plus1 != 0 && unit == 0 && leader && item + 1 == static_cast<uint32_t>(g.withhold_plus1);
        if (!withhold) {
          // (withheld, for a test of the failure path: this stage's barrier is
          // never armed, so the MMA issuer's bounded wait for it runs out)
          uint8_t* sa = stage_base + stage * kStageBytes;
          uint8_t* sb = sa + kABytes;
          const int k0 = kb * kBK;
          const int m0 = mb * C::kTileM + static_cast<int>(rank) * kBM;
          const int n0 = nb * kBN + static_cast<int>(rank) * C::kBRows;
          auto load = [&](void* dst, const CUtensorMap* map, int x, int y) {
            if constexpr (PAIR) {
              if (!leader) {
                tma_load_2d_pair(dst, map, map_to_rank(&full[stage], 0), x, y);
                return;
              }
            }
            tma_load_2d(dst, map, &full[stage], x, y);
          };
          auto load3 = [&](void* dst, const CUtensorMap* map, int y, int z) {
            if constexpr (PAIR) {
              if (!leader) {
                tma_load_3d_pair(dst, map, map_to_rank(&full[stage], 0), 0, y, z);
                return;
              }
            }
            tma_load_3d(dst, map, &full[stage], 0, y, z);
          };
          // the leader's stage barrier counts both CTAs' bytes
          if (leader) mbar_arrive_expect_tx(&full[stage], PAIR ? 2 * kStageBytes : kStageBytes);
          if (g.a_blocked) {
            if constexpr (A_MN) load3(sa, &tma_a, k0, m0 >> 6);  // blocks m0/64 and m0/64 + 1
            else load3(sa, &tma_a, m0, kb);
          } else if constexpr (A_MN) {
            load(sa, &tma_a, m0, k0);
            load(sa + 8192, &tma_a, m0 + 64, k0);
          } else {
            load(sa, &tma_a, k0, m0);
          }
          if constexpr (B_MN) {
#pragma unroll
            for (int j = 0; j < C::kBRows / 64; ++j) load(sb + j * 8192, &tma_b, n0 + 64 * j, k0);
          } else {
            load(sb, &tma_b, k0, n0);
          }
        }
        ++done;
        item += kProducers;
        for (int i = 0; i < kProducers && have; ++i) have = next_item();
      }
      if (*abort_flag) {
        // copies still in flight land before the CTA exits: the leader's stage
        // barriers count them (both CTAs' for a pair); a pair's other CTA
        // cannot see its own and waits out a fixed, generous interval instead
        if (leader) {
          const uint64_t t0 = global_timer_ns();
          for (uint32_t d = 0; d < done && d < static_cast<uint32_t>(kStages / kProducers); ++d) {
            const uint32_t n = item - kProducers * (d + 1);  // this producer's last loads
            const uint32_t a = smem_u32(&full[n % kStages]);
            while (!mbar_try_wait(a, (n / kStages) & 1, 20000u) && global_timer_ns() - t0 < wait_limit_ns()) {
            }
          }
        }
        if (PAIR) sleep_ns_bounded(200000);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (the leader of a pair) ----------------
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = instr_desc(C::kTileM, kBN, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool run = true;
      for (int tile = unit; tile < num_tiles_run && run; tile += units) {
        int mb, nb, ks, kb0, kb1;
        tile_coords(tile, mb, nb, ks);
        kb_range(ks, kb0, kb1);
        if (!wait_or_abort<PAIR>(&tmem_empty[acc], acc_phase ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kBN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!wait_or_abort<PAIR>(&full[stage], phase, abort_flag)) {
            run = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(stage_base + stage * kStageBytes);
          const uint32_t sb = sa + kABytes;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            // K-major: the 16-wide K step moves 32 bytes along the swizzled row;
            // M/N-major: it moves 16 rows (2 x 1024-byte swizzle atoms).
            const uint64_t ad = A_MN ? smem_desc(sa + k * 2048, 8192, 1024) : smem_desc(sa + k * 32, 16, 1024);
            const uint64_t bd = B_MN ? smem_desc(sb + k * 2048, 8192, 1024) : smem_desc(sb + k * 32, 16, 1024);
            umma_bf16<PAIR>(d_tmem, ad, bd, idesc, (kb != kb0 || k != 0) ? 1u : 0u);
          }
          umma_commit<PAIR>(&empty[stage]);  // stage free (in both CTAs) once these MMAs have read it
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!run) break;
        umma_commit<PAIR>(&tmem_full[acc]);  // accumulator complete
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      // every MMA issued has finished reading shared memory (both CTAs') and
      // writing TMEM before the teardown
      umma_commit<PAIR>(mma_done);
      (void)mbar_wait(mma_done, 0);
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int q = warp & 3;  // TMEM lane quarter this warp may access: rows 32q .. 32q + 31
    uint8_t* my_stage = out_stage + q * 2 * kStageOutBytes;
    int acc = 0;
    uint32_t acc_phase = 0;
    int nstore = 0;  // bulk groups committed by this warp (lane 0)
    for (int tile = unit; tile < num_tiles_run; tile += units) {
      int mb, nb, ks;
      tile_coords(tile, mb, nb, ks);
      const int rbase = mb * C::kTileM + static_cast<int>(rank) * kBM + q * 32;  // this warp's first row
      const int y = ks * g.split_rows + rbase;                                   // its first output row
      const int row = rbase + lane;  // this thread's row of the M rows
      // the cross-entropy epilogue's per-row inputs, loaded while the tile's MMAs run
      int64_t row_t = 0;
      float row_r = 0.0f;
      if (kLogits && g.epi == kEpiCeExp && row < g.M) {
        row_t = g.targets[row];
        if (g.row_ref) row_r = g.row_ref[row];
      }
      if (!wait_or_abort<PAIR>(&tmem_full[acc], acc_phase, abort_flag)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + acc * kBN + (static_cast<uint32_t>(q * 32) << 16);
      // 32 rows x 64 bf16 (this warp's slice at column x) to global memory
      // through a 128-byte swizzled staging buffer and one TMA store.
      // Slices go out in pairs (columns x and x + 64, staged in the warp's two
      // buffers): one proxy fence and one bulk group per pair, one copy of
      // both 64-column blocks for the blocked layout (box {64, 32, 2}).
      // Every tile stages an even number of slices.
      auto store_slice = [&](const uint32_t (&pk)[32], int x) {
        const int b = nstore & 1;
        if (b == 0 && nstore >= 2) {  // the previous pair's copy has read both buffers
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
        }
        uint8_t* rowp = my_stage + b * kStageOutBytes + lane * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(rowp + ((c ^ (lane & 7)) << 4)) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        if (b == 1) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (g.out_blocked) {
              // evict first: the chunk's exponentials are larger than L2 and
              // are read back only by the next kernels, after most of them have
              // left L2 anyway; the operands that tiles share stay
              tma_store_3d_hint(&tma_out, my_stage, 0, y, (x - 64) >> 6, l2_policy_evict_first());
            } else {
              tma_store_2d(&tma_out, my_stage, x - 64, y);
              tma_store_2d(&tma_out, my_stage + kStageOutBytes, x, y);
            }
            bulk_commit();
          }
        }
        ++nstore;
      };
      if (kLogits && g.epi == kEpiCeExp && g.N - nb * kBN >= kBN) {
        // A whole tile of the fused cross-entropy: every column is inside N.
        // exp(x - R) = 2^(x log2 e - R log2 e) with packed f32x2 arithmetic; a
        // reference of -inf stores 0 for rows that are ignored or past M.
        float nr = -INFINITY;
        int tcol = -1;
        if (row < g.M) {
          const int64_t t = row_t;
          if (t != g.ignore_index && t >= 0 && t < g.N) {
            nr = -row_r * kLog2e;
            const int64_t off = t - static_cast<int64_t>(nb) * kBN;
            if (off >= 0 && off < kBN) tcol = static_cast<int>(off);
          }
        }
        const float2 l2 = make_float2(kLog2e, kLog2e), n2 = make_float2(nr, nr);
        float2 sA = make_float2(0.f, 0.f), sB = make_float2(0.f, 0.f);
        float mA = -INFINITY, mB = -INFINITY;
        auto slice = [&](const uint32_t (&u0)[32], const uint32_t (&u1)[32], int cs) {
          if (tcol >= cs && tcol < cs + 64) {
            float xt = 0.f;
#pragma unroll
            for (int j = 0; j < 64; ++j)
              if (j == tcol - cs) xt = __uint_as_float(j < 32 ? u0[j] : u1[j - 32]);
            g.x_target[row] = xt;
          }
          uint32_t pk[32];
#pragma unroll
          for (int j = 0; j < 64; j += 4) {
            const uint32_t* u = j < 32 ? u0 : u1;
            const int i = j & 31;
            const float2 xa = make_float2(__uint_as_float(u[i]), __uint_as_float(u[i + 1]));
            const float2 xb = make_float2(__uint_as_float(u[i + 2]), __uint_as_float(u[i + 3]));
            const float2 ya = __ffma2_rn(xa, l2, n2);
            const float2 yb = __ffma2_rn(xb, l2, n2);
            const float2 ea = make_float2(ex2(ya.x), ex2(ya.y));
            const float2 eb = make_float2(ex2(yb.x), ex2(yb.y));
            sA = __fadd2_rn(sA, ea);
            sB = __fadd2_rn(sB, eb);
            mA = fmaxf(mA, fmaxf(xa.x, xa.y));
            mB = fmaxf(mB, fmaxf(xb.x, xb.y));
            pk[j / 2] = pack_bf16x2(ea.x, ea.y);
            pk[j / 2 + 1] = pack_bf16x2(eb.x, eb.y);
          }
          store_slice(pk, nb * kBN + cs);
        };
        // two register sets: one slice's TMEM loads fly while the other is processed
        uint32_t a0[32], a1[32], b0[32], b1[32];
        tmem_ld32(t_row, a0);
        tmem_ld32(t_row + 32, a1);
        tmem_ld_wait(a0, a1);
        tmem_ld32(t_row + 64, b0);
        tmem_ld32(t_row + 96, b1);
        slice(a0, a1, 0);
        tmem_ld_wait(b0, b1);
        tmem_ld32(t_row + 128, a0);
        tmem_ld32(t_row + 160, a1);
        slice(b0, b1, 64);
        tmem_ld_wait(a0, a1);
        tmem_ld32(t_row + 192, b0);
        tmem_ld32(t_row + 224, b1);
        slice(a0, a1, 128);
        tmem_ld_wait(b0, b1);
        slice(b0, b1, 192);
        if (row < g.M)
          g.stats[static_cast<int64_t>(nb) * g.stats_ld + row] =
              make_float2((sA.x + sA.y) + (sB.x + sB.y), fmaxf(mA, mB));
      } else if (g.epi == kEpiStoreBf16 || (kLogits && g.epi == kEpiCeExp)) {
        // The bf16 store (optionally row-scaled), and the fused cross-entropy's
        // last column tile, whose columns past N are left out of the sum and max.
        const bool ce = kLogits && g.epi == kEpiCeExp;
        float rs = 1.0f, nrl2 = 0.0f;
        int tcol = -1;       // target column relative to the tile (-1: none)
        bool keep = true;    // row stores its exponentials (valid row)
        if (ce) {
          keep = false;
          if (row < g.M) {
            const int64_t t = row_t;
            keep = t != g.ignore_index && t >= 0 && t < g.N;
            if (keep && t >= static_cast<int64_t>(nb) * kBN && t < static_cast<int64_t>(nb) * kBN + kBN)
              tcol = static_cast<int>(t - static_cast<int64_t>(nb) * kBN);
            nrl2 = -row_r * kLog2e;
          }
        } else if (g.row_scale) {
          rs = row < g.M ? g.row_scale[row] : 0.0f;
        }
        const int cols_left = g.N - nb * kBN;  // columns of this tile inside N
        float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
        float m0 = -INFINITY, m1 = -INFINITY;
        // 64-column slices: 2 TMEM loads -> 32 rows x 128 bytes, 128-byte swizzled.
        // The next slice's TMEM loads are in flight while this one is processed.
        uint32_t n0[32], n1[32];
        tmem_ld32(t_row, n0);
        tmem_ld32(t_row + 32, n1);
        tmem_ld_wait(n0, n1);
#pragma unroll 1
        for (int cs = 0; cs < kBN; cs += 64) {
          uint32_t v0[32], v1[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            v0[j] = n0[j];
            v1[j] = n1[j];
          }
          if (cs + 64 < kBN) {
            tmem_ld32(t_row + cs + 64, n0);
            tmem_ld32(t_row + cs + 96, n1);
          }
          if (ce) {
            if (tcol >= cs && tcol < cs + 64) {
              float xt = 0.f;
#pragma unroll
              for (int j = 0; j < 64; ++j)
                if (j == tcol - cs) xt = __uint_as_float(j < 32 ? v0[j] : v1[j - 32]);
              g.x_target[row] = xt;
            }
            const bool whole = cols_left >= cs + 64;
#pragma unroll
            for (int j = 0; j < 64; ++j) {
              uint32_t& w = j < 32 ? v0[j] : v1[j - 32];
              const float x = __uint_as_float(w);
              float e = 0.0f;
              if (whole || cs + j < cols_left) {
                e = ex2(fmaf(x, kLog2e, nrl2));
                if (j & 1) m1 = fmaxf(m1, x); else m0 = fmaxf(m0, x);
                switch (j & 3) {
                  case 0: s0 += e; break;
                  case 1: s1 += e; break;
                  case 2: s2 += e; break;
                  default: s3 += e; break;
                }
              }
              w = __float_as_uint(keep ? e : 0.0f);
            }
          } else if (g.row_scale) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              v0[j] = __float_as_uint(__uint_as_float(v0[j]) * rs);
              v1[j] = __float_as_uint(__uint_as_float(v1[j]) * rs);
            }
          }
          uint32_t pk[32];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            pk[j / 2] = pack_bf16x2(__uint_as_float(v0[j]), __uint_as_float(v0[j + 1]));
            pk[16 + j / 2] = pack_bf16x2(__uint_as_float(v1[j]), __uint_as_float(v1[j + 1]));
          }
          store_slice(pk, nb * kBN + cs);
          if (cs + 64 < kBN) tmem_ld_wait(n0, n1);
        }
        if (ce && row < g.M)
          g.stats[static_cast<int64_t>(nb) * g.stats_ld + row] =
              make_float2((s0 + s1) + (s2 + s3), fmaxf(m0, m1));
      } else if (kDw && g.epi == kEpiAccToBf16) {
        // Each 64-column slice: the fp32 accumulator's 32 rows come in by TMA
        // (two 32-column boxes, one per staging buffer, zeros outside the
        // map), the tile is added, the sum rounded once to bf16 and stored by
        // TMA from the first buffer (clipped outside the map).
#pragma unroll 1
        for (int cs = 0; cs < kBN; cs += 64) {
          const int n = nstore;
          uint64_t* bar = &epi_bar[2 * q];
          if (lane == 0) {
            bulk_wait_read_all();  // the previous slice's store has read the first buffer
            mbar_arrive_expect_tx(bar, 2 * kStageOutBytes);
            tma_load_2d(my_stage, &tma_aux, bar, nb * kBN + cs, y);
            tma_load_2d(my_stage + kStageOutBytes, &tma_aux, bar, nb * kBN + cs + 32, y);
          }
          __syncwarp();
          uint32_t v0[32], v1[32];
          tmem_ld32(t_row + cs, v0);
          tmem_ld32(t_row + cs + 32, v1);
          tmem_ld_wait(v0, v1);
          if (!__all_sync(0xffffffffu, wait_or_abort<false>(bar, n & 1, abort_flag))) {
            if (lane == 0) {  // the two loads land before the CTA exits
              const uint64_t t0 = global_timer_ns();
              while (!mbar_try_wait(smem_u32(bar), n & 1, 20000u) && global_timer_ns() - t0 < wait_limit_ns()) {
              }
            }
            __syncwarp();
            break;
          }
          uint8_t* rowp = my_stage + lane * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float4 a = *reinterpret_cast<const float4*>(rowp + ((c ^ (lane & 7)) << 4));
            const float4 b = *reinterpret_cast<const float4*>(rowp + kStageOutBytes + ((c ^ (lane & 7)) << 4));
            v0[4 * c] = __float_as_uint(__uint_as_float(v0[4 * c]) + a.x);
            v0[4 * c + 1] = __float_as_uint(__uint_as_float(v0[4 * c + 1]) + a.y);
            v0[4 * c + 2] = __float_as_uint(__uint_as_float(v0[4 * c + 2]) + a.z);
            v0[4 * c + 3] = __float_as_uint(__uint_as_float(v0[4 * c + 3]) + a.w);
            v1[4 * c] = __float_as_uint(__uint_as_float(v1[4 * c]) + b.x);
            v1[4 * c + 1] = __float_as_uint(__uint_as_float(v1[4 * c + 1]) + b.y);
            v1[4 * c + 2] = __float_as_uint(__uint_as_float(v1[4 * c + 2]) + b.z);
            v1[4 * c + 3] = __float_as_uint(__uint_as_float(v1[4 * c + 3]) + b.w);
          }
          // this row's 64 bf16 over its own 128 bytes of the first buffer
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint32_t* t = c < 4 ? &v0[8 * c] : &v1[8 * (c - 4)];
            *reinterpret_cast<uint4*>(rowp + ((c ^ (lane & 7)) << 4)) =
                make_uint4(pack_bf16x2(__uint_as_float(t[0]), __uint_as_float(t[1])),
                           pack_bf16x2(__uint_as_float(t[2]), __uint_as_float(t[3])),
                           pack_bf16x2(__uint_as_float(t[4]), __uint_as_float(t[5])),
                           pack_bf16x2(__uint_as_float(t[6]), __uint_as_float(t[7])));
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tma_out, my_stage, nb * kBN + cs, y);
            bulk_commit();
          }
          ++nstore;
        }
      } else if (!kLogits && (g.epi == kEpiStoreF32 || g.epi == kEpiAddF32)) {
        // 32-column slices: 1 TMEM load -> 32 rows x 128 bytes of fp32
        const float rs = g.row_scale ? (row < g.M ? g.row_scale[row] : 0.0f) : 1.0f;
#pragma unroll 1
        for (int cs = 0; cs < kBN; cs += 32) {
          uint32_t v[32];
          tmem_ld32(t_row + cs, v);
          tmem_ld_wait(v);
          if (g.row_scale) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * rs);
          }
          uint8_t* buf = my_stage + (nstore & 1) * kStageOutBytes;
          if (nstore >= 2) {
            if (lane == 0) bulk_wait_read_1();
            __syncwarp();
          }
          uint8_t* rowp = buf + lane * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(rowp + ((c ^ (lane & 7)) << 4)) =
                make_uint4(v[c * 4], v[c * 4 + 1], v[c * 4 + 2], v[c * 4 + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (g.epi == kEpiStoreF32) tma_store_2d(&tma_out, buf, nb * kBN + cs, y);
            else tma_reduce_add_2d(&tma_out, buf, nb * kBN + cs, y);
            bulk_commit();
          }
          ++nstore;
        }
      } else if (kDw) {
        // kEpiBf16Add: each 64-column slice of the warp's 32 output rows comes
        // in by TMA (zeros outside the map) into a staging buffer, gets the
        // tile added in place, rounded once to bf16, and goes back out by TMA
        // (clipped outside the map).  The next slice's load flies while this
        // slice is added.
        auto issue = [&](int n, int x) {  // the warp's n-th slice, into buffer n & 1
          if (lane == 0) {
            uint64_t* bar = &epi_bar[2 * q + (n & 1)];
            mbar_arrive_expect_tx(bar, kStageOutBytes);
            tma_load_2d(my_stage + (n & 1) * kStageOutBytes, &tma_out, bar, x, y);
          }
        };
        // a buffer is free once the store that used it has read it: two
        // slices back for the first slice, one back for the next
        if (lane == 0) bulk_wait_read_1();
        __syncwarp();
        issue(nstore, nb * kBN);
        bool ok = true;
#pragma unroll 1
        for (int cs = 0; cs < kBN; cs += 64) {
          const int n = nstore;
          const bool next = cs + 64 < kBN;
          if (next) {
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
            issue(n + 1, nb * kBN + cs + 64);
          }
          uint32_t v0[32], v1[32];
          tmem_ld32(t_row + cs, v0);
          tmem_ld32(t_row + cs + 32, v1);
          tmem_ld_wait(v0, v1);
          ok = __all_sync(0xffffffffu, wait_or_abort<false>(&epi_bar[2 * q + (n & 1)], (n >> 1) & 1, abort_flag));
          if (!ok) {
            // the loads this warp issued land before the CTA exits
            if (lane == 0) {
              const uint64_t t0 = global_timer_ns();
              for (int m = n; m <= n + (next ? 1 : 0); ++m) {
                const uint32_t a = smem_u32(&epi_bar[2 * q + (m & 1)]);
                while (!mbar_try_wait(a, (m >> 1) & 1, 20000u) && global_timer_ns() - t0 < wait_limit_ns()) {
                }
              }
            }
            __syncwarp();
            break;
          }
          uint8_t* buf = my_stage + (n & 1) * kStageOutBytes;
          uint8_t* rowp = buf + lane * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint4* p = reinterpret_cast<uint4*>(rowp + ((c ^ (lane & 7)) << 4));
            const uint4 prev = *p;
            const uint32_t* t = c < 4 ? &v0[8 * c] : &v1[8 * (c - 4)];
            *p = make_uint4(pack_bf16x2(bf16_lo(prev.x) + __uint_as_float(t[0]), bf16_hi(prev.x) + __uint_as_float(t[1])),
                            pack_bf16x2(bf16_lo(prev.y) + __uint_as_float(t[2]), bf16_hi(prev.y) + __uint_as_float(t[3])),
                            pack_bf16x2(bf16_lo(prev.z) + __uint_as_float(t[4]), bf16_hi(prev.z) + __uint_as_float(t[5])),
                            pack_bf16x2(bf16_lo(prev.w) + __uint_as_float(t[6]), bf16_hi(prev.w) + __uint_as_float(t[7])));
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tma_out, buf, nb * kBN + cs, y);
            bulk_commit();
          }
          ++nstore;
        }
        if (!ok) break;
      }
      // every TMEM load of this accumulator is complete: hand it back to the MMA
      // warp (of the pair's leader)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR) mbar_arrive_cluster(map_to_rank(&tmem_empty[acc], 0));
        else mbar_arrive(&tmem_empty[acc]);
      }
      if (kDx && g.epi == kEpiStoreF32 && g.k_splits > 1 && g.split_out) {
        // this warp's partial rows are written (not only read out of shared
        // memory) before the slice's count goes up
        if (lane == 0) bulk_wait_all();
        __syncwarp();
        const int cidx = ((mb * g.tiles_n + nb) * (PAIR ? 2 : 1) + static_cast<int>(rank)) * 4 + q;
        // rows r0, r0 + rstep, ... of the slice are summed by this warp
        int r0 = 0, rstep = 1;
        int go = 0;
        if (lane == 0) {
          __threadfence();
          const int before = atomicAdd(&g.split_count[cidx], 1);
          if (g.split_target > 0) {
            // every split's warp waits for the others, then takes its share of the rows
            const volatile int* cnt = &g.split_count[cidx];
            const uint64_t t0 = global_timer_ns();
            go = 1;
            while (*cnt < g.split_target) {
              if (global_timer_ns() - t0 > wait_limit_ns()) {
                record_status(GH_ERR_TIMEOUT);
                go = 0;
                break;
              }
              __nanosleep(64);
            }
          } else {
            go = before == g.k_splits - 1;  // the last split sums the whole slice
            if (go) g.split_count[cidx] = 0;
          }
        }
        go = __shfl_sync(0xffffffffu, go, 0);
        if (g.split_target > 0) {
          r0 = ks;
          rstep = g.k_splits;
        }
        if (go) {
          __threadfence();  // every split's partial of this slice is visible
          const int col = nb * kBN + 8 * lane;  // lanes across the row: coalesced 32-byte reads
          if (col < g.N) {
            // 2 rows at a time with every split's loads issued before the adds
#pragma unroll 1
            for (int r = r0; r < 32; r += 2 * rstep) {
              float4 u[kMaxSplits][2][2];
#pragma unroll
              for (int sp = 0; sp < kMaxSplits; ++sp) {
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                  const int rr = rbase + r + i * rstep;
                  if (sp < g.k_splits && r + i * rstep < 32 && rr < g.M) {
                    const float* p = g.split_ws + (static_cast<int64_t>(sp) * g.split_rows + rr) * g.N + col;
                    u[sp][i][0] = __ldcg(reinterpret_cast<const float4*>(p));
                    u[sp][i][1] = __ldcg(reinterpret_cast<const float4*>(p + 4));
                  }
                }
              }
#pragma unroll
              for (int i = 0; i < 2; ++i) {
                const int rr = rbase + r + i * rstep;
                if (r + i * rstep >= 32 || rr >= g.M) break;
                float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int sp = 0; sp < kMaxSplits; ++sp) {
                  if (sp < g.k_splits) {
                    a[0] += u[sp][i][0].x; a[1] += u[sp][i][0].y; a[2] += u[sp][i][0].z; a[3] += u[sp][i][0].w;
                    a[4] += u[sp][i][1].x; a[5] += u[sp][i][1].y; a[6] += u[sp][i][1].z; a[7] += u[sp][i][1].w;
                  }
                }
                *reinterpret_cast<uint4*>(g.split_out + static_cast<int64_t>(rr) * g.split_ld + col) =
                    make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]), pack_bf16x2(a[4], a[5]),
                               pack_bf16x2(a[6], a[7]));
              }
            }
          }
        }
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    if (lane == 0) bulk_wait_all();  // staging buffers stay valid until the stores have read them
  }

  // ---------------- teardown ----------------
  __syncwarp();
  if (g.defer_wait) pdl_wait();  // complete only after the previous kernel
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) {  // neither CTA leaves while the other may still signal it or read its tiles
    cluster_arrive_release();
    cluster_wait_acquire();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<PAIR>(tmem_base, kTmemCols);
  }
}

}  // namespace sm100
}  // namespace gh
