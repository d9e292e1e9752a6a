// Chunked linear cross-entropy (Greyhound `chunked_linear_cross_entropy` over
// `chunked_linear_loss`): logits = X @ W^T are formed one row chunk at a time
// and never materialised in full.  Per chunk c (rows [c0, c0 + rows)):
//
//   1  P      = exp(X_c W^T - R)      tcgen05 GEMM whose epilogue turns the fp32
//                                     logits tile into bf16 exponentials P (0 for
//                                     ignored rows) and keeps, per (row, 256-column
//                                     tile), the sum of the exponentials, the max
//                                     logit and the target logit (R = 0)
//   2  finalize                       per row: lse, the row loss, the factor
//                                     alpha = scale (1 + 2 z lse) exp(R - lse),
//                                     the target element P[t] -= scale / alpha and
//                                     Xs_c = bf16(alpha X_c); then the logits
//                                     gradient is exactly G_c = diag(alpha) P
//   3  (recompute)                    only when a row's lse fell outside
//                                     [-40, 40], where exp(x) is not safe in
//                                     fp32/bf16: steps 1 and 2 again with R = the
//                                     row's max logit (both launches exit at once
//                                     when no row asked for it)
//   4  dX_c   = diag(alpha) (P W)     tcgen05 GEMM (A K-major, B N-major), the
//                                     row factor applied in its epilogue
//   5  dW    (+)= P^T Xs_c            tcgen05 GEMM (both operands M/N-major);
//                                     fp32 accumulator across chunks (TMA store,
//                                     then TMA reduce-add in L2; the last chunk
//                                     adds it and rounds once to bf16, "fp32"),
//                                     or accumulated in the bf16 output ("weight")
// When the dX tiles alone would leave SMs idle, dX splits K into fp32 partials;
// inside the same kernel the last split to finish each 32-row slice sums them in
// split order (deterministic) and writes the bf16 rows.  With fp32 accumulation
// the last chunk's dW epilogue adds the accumulator and rounds once to bf16.
//
// gh_chunked_linear_loss (a caller-provided loss per chunk) keeps the plain
// form: step 1 stores the bf16 logits, the caller's callback overwrites them
// with its gradient G_c, and steps 4-5 run with alpha = 1 and X_c.
//
// The loss is the fixed-order sum of all rows' losses, divided by the valid
// count for "mean".  ld = round_up(V, 8) keeps chunk rows 16-byte aligned as
// TMA requires; TMA reads the chunk with extent V, so its padding columns are
// never used.
#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "ce.h"
#include "common.cuh"
#include "gemm_sm100.cuh"
#include "linear_ce.h"
#include "profile.h"

namespace gh {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// 2-D tensor map: `inner` contiguous elements per row, `outer` rows of
// `row_bytes`, box {box_inner, box_outer}, 128-byte swizzle, zero fill
// outside (loads) / clipping (stores).
bool make_tmap(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
               uint32_t box_outer, bool f32 = false, uint32_t box_inner = 64) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
             dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map of a chunk's exponentials P in the column-blocked layout: element
// (row r, column c) at ((c / 64) * blk_rows + r) * 64 + c % 64, dims {64, rows,
// nblk}, box {64, box_rows, box_blocks}, 128-byte swizzle.  A box of whole
// 64-column blocks is contiguous memory, and no box reaches past the array.
bool make_pblk(CUtensorMap* m, const void* base, uint64_t rows, uint64_t nblk, uint64_t blk_rows, uint32_t box_rows,
               uint32_t box_blocks) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {64, rows, nblk};
  const cuuint64_t strides[2] = {128, blk_rows * 128};
  const cuuint32_t box[3] = {64, box_rows, box_blocks};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output maps of the GEMM epilogue: 32-row boxes of 128 bytes (64 bf16 or 32 fp32).
bool make_out_bf16(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t ld) {
  return make_tmap(m, base, cols, rows, ld * 2, 32, false, 64);
}
bool make_out_f32(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t ld) {
  return make_tmap(m, base, cols, rows, ld * 4, 32, true, 32);
}

// Per-chunk step 2 of the fused cross-entropy (one CTA of 512 threads per 32
// rows).  Each row's statistics are combined over the column tiles in a fixed
// order (deterministic): S = sum of the tiles' sums of exp(x - R), M = max.
struct FinalizeArgs {
  const float2* stats;      // [tiles_n][stats_ld]
  int stats_ld, tiles_n;
  const int64_t* targets;   // chunk rows
  int64_t ignore_index;
  int V, rows, D;
  float z;
  int mean;
  const unsigned long long* n_valid;
  const float* x_target;    // [rows] fp32 target logits
  float* row_max;           // [rows]: written by the first pass, the recompute's R
  int recompute;            // 0: first pass (R = 0); 1: recompute (R = row_max)
  int* flag;                // first pass: set when a row needs the recompute; recompute: runs only if set
  float* alpha;             // [rows]
  float* row_loss;          // [rows] (this chunk's slice)
  uint16_t* P;              // exponentials of the chunk, column-blocked (blocks of blk_rows x 64)
  int64_t blk_rows;
  const uint16_t* X;        // [rows, D] inputs of the chunk
  uint16_t* Xs;             // [rows, D] alpha-scaled inputs
};

// exp(x) with R = 0 is exact to fp32 rounding and neither overflows nor loses
// the row to underflow while the row's lse stays within this window.
constexpr float kLseWindow = 40.0f;
// |1 + 2 z lse| is raised to at least this value, so scale / alpha stays finite;
// the gradient entries this changes are below scale * 2^-20 (the bf16 rounding
// of the target entry alone is scale * 2^-9).
constexpr float kZFactorFloor = 9.5367431640625e-07f;  // 2^-20

constexpr int kFinWarps = 16;

__global__ void __launch_bounds__(kFinWarps * 32) lce_finalize_kernel(FinalizeArgs a) {
  __shared__ float sh_s[kFinWarps][32];
  __shared__ float sh_m[kFinWarps][32];
  __shared__ float sh_alpha[32];
  pdl_wait();
  pdl_trigger();
  if (a.recompute && *reinterpret_cast<const volatile int*>(a.flag) == 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * 32;
  const int row = row0 + lane;
  float s = 0.0f, m = -INFINITY;
  if (row < a.rows) {
#pragma unroll 4
    for (int nb = warp; nb < a.tiles_n; nb += kFinWarps) {
      const float2 v = a.stats[static_cast<int64_t>(nb) * a.stats_ld + row];
      s += v.x;
      m = fmaxf(m, v.y);
    }
  }
  sh_s[warp][lane] = s;
  sh_m[warp][lane] = m;
  __syncthreads();
  if (warp == 0) {
    float alpha = 0.0f;
    if (row < a.rows) {
      float S = 0.0f, M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kFinWarps; ++w) {
        S += sh_s[w][lane];
        M = fmaxf(M, sh_m[w][lane]);
      }
      const int64_t t = a.targets[row];
      const bool valid = t != a.ignore_index && t >= 0 && t < a.V;
      const float R = a.recompute ? a.row_max[row] : 0.0f;
      if (!a.recompute) a.row_max[row] = M;
      float loss = 0.0f;
      if (valid) {
        const float lse = R + logf(S);
        const bool ok = a.recompute || (lse >= -kLseWindow && lse <= kLseWindow);
        if (!ok) {
          atomicExch(a.flag, 1);  // this chunk runs the recompute; its outputs come from there
        } else {
          float f = fmaf(2.0f * a.z, lse, 1.0f);
          if (!(fabsf(f) >= kZFactorFloor)) f = f < 0.0f ? -kZFactorFloor : kZFactorFloor;
          const unsigned long long nv = *a.n_valid;
          const float scale = a.mean ? 1.0f / static_cast<float>(nv > 0 ? nv : 1ull) : 1.0f;
          const float xt = a.x_target[row];
          alpha = scale * f * expf(R - lse);
          loss = (lse - xt) + a.z * lse * lse;
          // G[t] = alpha (exp(x_t - R) - scale / alpha) = scale ((1 + 2 z lse) p_t - 1)
          a.P[((t >> 6) * a.blk_rows + row) * 64 + (t & 63)] = to_bf16_bits(expf(xt - R) - scale / alpha);
        }
      }
      a.row_loss[row] = loss;
      a.alpha[row] = alpha;
    }
    sh_alpha[lane] = alpha;
  }
  __syncthreads();
  // Xs = bf16(alpha X) for this block's rows, 16-byte vectors
  const int d8 = a.D / 8;
  const int nrows = min(32, a.rows - row0);
  for (int i = threadIdx.x; i < nrows * d8; i += kFinWarps * 32) {
    const int r = i / d8, c = i - r * d8;
    const int64_t off = static_cast<int64_t>(row0 + r) * a.D + 8 * c;
    const uint4 x = *reinterpret_cast<const uint4*>(a.X + off);
    const float al = sh_alpha[r];
    *reinterpret_cast<uint4*>(a.Xs + off) =
        make_uint4(pack_bf16x2(bf16_lo(x.x) * al, bf16_hi(x.x) * al), pack_bf16x2(bf16_lo(x.y) * al, bf16_hi(x.y) * al),
                   pack_bf16x2(bf16_lo(x.z) * al, bf16_hi(x.z) * al), pack_bf16x2(bf16_lo(x.w) * al, bf16_hi(x.w) * al));
  }
}

__global__ void cast_f32_bf16_kernel(const float* __restrict__ src, int64_t n, uint16_t* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const int64_t n4 = n / 4;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4; i += stride) {
    const float4 v = reinterpret_cast<const float4*>(src)[i];
    reinterpret_cast<uint2*>(out)[i] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  }
  for (int64_t i = 4 * n4 + blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n; i += stride)
    out[i] = to_bf16_bits(src[i]);
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

// Tiles of the three GEMMs go to CTA pairs (cta_group::2, 256 x 256 tiles) by
// default; GH_GEMM=single selects one CTA per 128 x 256 tile (tests,
// measurements).
bool use_pairs() {
  const char* e = std::getenv("GH_GEMM");
  return !(e && std::strcmp(e, "single") == 0);
}

template <bool A_MN, bool B_MN>
gh_status_t launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tout,
                        const sm100::GemmArgs& g, bool pair, int kind, cudaStream_t stream,
                        const CUtensorMap* taux = nullptr, int max_sms = 0) {
  // taux: the fp32 accumulator read by kEpiAccToBf16 (any valid map otherwise);
  // max_sms > 0: the launch uses at most that many SMs
  const CUtensorMap& tx = taux ? *taux : tout;
  const int sms = max_sms > 0 ? std::min(max_sms, sm_count()) : sm_count();
  const int tiles = g.tiles_m * g.tiles_n * g.k_splits;
  if (tiles == 0) return GH_OK;
  sm100::GemmArgs ga = g;
  if (!g.run_flag) ga.withhold_plus1 = static_cast<int>(debug_gemm_stage().exchange(-1) + 1);
  cudaError_t e;
  if (pair) {
    auto kern = sm100::gemm_bf16_kernel<A_MN, B_MN, true>;
    if (ensure_smem_limit(kern, sm100::GemmCfg<true>::kSmem) != cudaSuccess) return GH_ERR_CUDA;
    const int pairs = std::min(tiles, std::max(1, sms / 2));
    ProfileScope prof(kind, stream);
    e = launch_pdl(kern, dim3(2 * pairs), dim3(sm100::kGemmThreads), sm100::GemmCfg<true>::kSmem, stream, 2, ta, tb,
                   tout, tx, ga);
  } else {
    auto kern = sm100::gemm_bf16_kernel<A_MN, B_MN, false>;
    if (ensure_smem_limit(kern, sm100::GemmCfg<false>::kSmem) != cudaSuccess) return GH_ERR_CUDA;
    const int grid = std::min(tiles, std::max(1, sms));
    ProfileScope prof(kind, stream);
    e = launch_pdl(kern, dim3(grid), dim3(sm100::kGemmThreads), sm100::GemmCfg<false>::kSmem, stream, 1, ta, tb,
                   tout, tx, ga);
  }
  note_launch();
  return e == cudaSuccess ? GH_OK : GH_ERR_CUDA;
}

sm100::GemmArgs gemm_args(int M, int N, int K, int m_fastest, int epi, bool pair) {
  const int tile_m = pair ? sm100::GemmCfg<true>::kTileM : sm100::GemmCfg<false>::kTileM;
  sm100::GemmArgs g{};
  g.M = M;
  g.N = N;
  g.K = K;
  g.tiles_m = (M + tile_m - 1) / tile_m;
  g.tiles_n = (N + sm100::kBN - 1) / sm100::kBN;
  g.num_kb = (K + sm100::kBK - 1) / sm100::kBK;
  g.k_splits = 1;
  g.kb_per_split = g.num_kb;
  g.m_fastest = m_fastest;
  g.epi = epi;
  return g;
}

// K splits for a long-K GEMM: the split count (at most max_splits, each split
// at least 16 K steps) that minimises (waves of work units) x (K steps per
// unit), when that saves at least 3% over no split.  It fills SMs that the
// output tiles alone would leave idle, and evens out a last wave of tiles
// that would run part-empty.
int choose_splits(int tiles, int num_kb, int units, int max_splits) {
  int best = 1;
  const int64_t base = (static_cast<int64_t>(tiles) + units - 1) / units * num_kb;
  int64_t best_cost = base;
  const int smax = std::min(max_splits, std::max(1, num_kb / 16));
  for (int sp = 2; sp <= smax; ++sp) {
    const int per = (num_kb + sp - 1) / sp;
    const int used = (num_kb + per - 1) / per;
    const int64_t waves = (static_cast<int64_t>(tiles) * used + units - 1) / units;
    const int64_t cost = waves * per;
    if (cost < best_cost && cost * 100 <= base * 97) {
      best_cost = cost;
      best = used;
    }
  }
  return best;
}

int64_t default_chunk(int64_t N, int64_t ld) {
  // Largest multiple of 128 rows whose bf16 chunk logits fit in 1 GiB, capped at N.
  int64_t c = ((int64_t(1) << 30) / (ld * 2)) / 128 * 128;
  c = std::max<int64_t>(c, 128);
  return std::min<int64_t>(c, std::max<int64_t>(N, 1));
}

}  // namespace

gh_status_t cast_f32_bf16_launch(const float* src, void* out, int64_t n, cudaStream_t stream) {
  if (n == 0) return GH_OK;
  const int64_t blocks = std::min<int64_t>((n / 4 + 255) / 256 + 1, static_cast<int64_t>(sm_count()) * 8);
  const cudaError_t e = launch_pdl(cast_f32_bf16_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream, 1,
                                   src, n, static_cast<uint16_t*>(out));
  note_launch();
  return e == cudaSuccess ? GH_OK : GH_ERR_CUDA;
}

gh_status_t linear_ce_run(const LinearCeArgs& a, cudaStream_t stream) {
  const int64_t N = a.N, D = a.D, V = a.V;
  if (N == 0) {
    // No token: zero loss, zero weight gradient.
    if (cudaMemsetAsync(a.loss, 0, sizeof(float), stream) != cudaSuccess) return GH_ERR_CUDA;
    if (a.dW32) {
      if (cudaMemsetAsync(a.dW32, 0, static_cast<size_t>(V) * D * 4, stream) != cudaSuccess) return GH_ERR_CUDA;
      if (a.on_slice) return a.on_slice(a.slice_ctx, 0, V, stream);
    } else if (cudaMemsetAsync(a.dW, 0, static_cast<size_t>(V) * D * 2, stream) != cudaSuccess) {
      return GH_ERR_CUDA;
    }
    return GH_OK;
  }
  if (!tensor_map_encoder()) return GH_ERR_UNSUPPORTED;
  const int64_t ld = (V + 7) / 8 * 8;
  int64_t chunk = a.chunk > 0 ? std::min<int64_t>(a.chunk, N) : default_chunk(N, ld);
  const int64_t nchunks = (N + chunk - 1) / chunk;
  if (chunk > INT32_MAX / 2 || V > INT32_MAX / 2) return GH_ERR_UNSUPPORTED;
  const bool custom = a.loss_fn != nullptr;
  const bool fused = !custom;  // the cross-entropy in the logits GEMM's epilogue
  // fp32 accumulation on the fused path: the weight gradient of two consecutive
  // chunks in one contraction (K = both chunks' rows), so the fp32 accumulator
  // is read and written half as often; the two chunks' exponentials and scaled
  // inputs sit side by side (chunk 2k in rows [0, chunk), 2k + 1 after it).
  // Only while the pair's scaled inputs (the B operand every tile of the
  // contraction reads) stay well inside L2: at 67 MB (the Llama-3-8B head) the
  // pair contraction re-read them from DRAM and the step's DRAM traffic grew
  // by a third.
  constexpr int64_t kPairDwMaxBytes = int64_t(32) << 20;
  const int grp = (fused && a.accum == GH_ACCUM_FP32 && nchunks > 1 && 2 * chunk * D * 2 <= kPairDwMaxBytes) ? 2 : 1;
  const int64_t ngroups = (nchunks + grp - 1) / grp;
  const int64_t blk_rows = grp * chunk;  // rows of one 64-column block of the exponentials
  // fp32 accumulator: library scratch when several weight-gradient contractions
  // must be summed before the single rounding, or the caller's fp32 output
  // (dW32: no rounding here)
  const bool out32 = a.dW32 != nullptr;
  const bool acc32 = !out32 && a.accum == GH_ACCUM_FP32 && ngroups > 1;
  const bool pair = use_pairs();
  const int tile_m = pair ? sm100::GemmCfg<true>::kTileM : sm100::GemmCfg<false>::kTileM;
  const int sms = sm_count();
  const int units = pair ? std::max(1, sms / 2) : sms;  // tile-processing units (CTA pairs or CTAs)
  const int tiles_m_max = static_cast<int>((chunk + tile_m - 1) / tile_m);
  const int dx_num_kb = static_cast<int>((V + sm100::kBK - 1) / sm100::kBK);
  const int dx_tiles_max = tiles_m_max * static_cast<int>((D + sm100::kBN - 1) / sm100::kBN);
  const int dx_splits = choose_splits(dx_tiles_max, dx_num_kb, units, sm100::kMaxSplits);
  const int64_t rows_pad = static_cast<int64_t>(tiles_m_max) * tile_m;

  const int tiles_n_logits = static_cast<int>((V + sm100::kBN - 1) / sm100::kBN);

  // scratch: [counter | row losses | chunk buffer | fp32 dW accumulator | dX split partials |
  //           fused only: tile statistics | target logits | row max | alpha | scaled inputs | flags]
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t off_rows = 256;
  const size_t off_buf = up(off_rows + sizeof(float) * N);
  // the chunk buffer: caller-visible row-major logits [chunk, ld] on the
  // plain path; the exponentials in 64-column blocks on the fused path
  const int64_t nblk = (V + 63) / 64;
  const size_t buf_bytes = static_cast<size_t>(fused ? blk_rows * nblk * 64 : chunk * ld) * 2;
  const size_t off_acc = up(off_buf + buf_bytes);
  const size_t acc_bytes = acc32 ? static_cast<size_t>(V) * D * 4 : 0;
  const size_t off_ws = up(off_acc + acc_bytes);
  const size_t ws_bytes = dx_splits > 1 ? static_cast<size_t>(dx_splits) * rows_pad * D * 4 : 0;
  const size_t off_stats = up(off_ws + ws_bytes);
  const size_t stats_bytes = fused ? static_cast<size_t>(tiles_n_logits) * rows_pad * sizeof(float2) : 0;
  const size_t off_xt = up(off_stats + stats_bytes);
  const size_t vec_bytes = fused ? static_cast<size_t>(rows_pad) * sizeof(float) : 0;
  const size_t off_rmax = up(off_xt + vec_bytes);
  const size_t off_alpha = up(off_rmax + vec_bytes);
  const size_t off_xs = up(off_alpha + vec_bytes);
  const size_t xs_bytes = fused ? static_cast<size_t>((grp - 1) * chunk + rows_pad) * D * 2 : 0;
  const size_t off_flags = up(off_xs + xs_bytes);
  const size_t flags_bytes = fused ? static_cast<size_t>(nchunks) * sizeof(int) : 0;
  const size_t off_count = up(off_flags + flags_bytes);
  const size_t count_bytes =
      dx_splits > 1 ? static_cast<size_t>(dx_tiles_max) * 2 /*CTAs of a pair*/ * 4 /*slices*/ * sizeof(int) : 0;
  const size_t total = off_count + count_bytes;
  void* scratch = nullptr;
  gh_status_t st = scratch_alloc(&scratch, total, stream);
  if (st != GH_OK) return st;
  char* base = static_cast<char*>(scratch);
  unsigned long long* counter = reinterpret_cast<unsigned long long*>(base);
  const unsigned long long* n_valid = a.n_total ? a.n_total : counter;
  float* row_loss = reinterpret_cast<float*>(base + off_rows);
  uint16_t* L = reinterpret_cast<uint16_t*>(base + off_buf);
  float* acc = acc32 ? reinterpret_cast<float*>(base + off_acc) : out32 ? a.dW32 : nullptr;
  float* ws = dx_splits > 1 ? reinterpret_cast<float*>(base + off_ws) : nullptr;
  float2* stats = fused ? reinterpret_cast<float2*>(base + off_stats) : nullptr;
  float* x_target = fused ? reinterpret_cast<float*>(base + off_xt) : nullptr;
  float* row_max = fused ? reinterpret_cast<float*>(base + off_rmax) : nullptr;
  float* alpha = fused ? reinterpret_cast<float*>(base + off_alpha) : nullptr;
  uint16_t* Xs = fused ? reinterpret_cast<uint16_t*>(base + off_xs) : nullptr;
  int* flags = fused ? reinterpret_cast<int*>(base + off_flags) : nullptr;
  int* split_count = dx_splits > 1 ? reinterpret_cast<int*>(base + off_count) : nullptr;

  const uint16_t* X = static_cast<const uint16_t*>(a.X);
  const uint16_t* W = static_cast<const uint16_t*>(a.W);
  uint16_t* dX = static_cast<uint16_t*>(a.dX);
  uint16_t* dW = static_cast<uint16_t*>(a.dW);

  st = custom    ? (cudaMemsetAsync(a.loss, 0, sizeof(float), stream) == cudaSuccess ? GH_OK : GH_ERR_CUDA)
       : a.n_total ? GH_OK
                   : ce_count_launch(a.targets, N, V, a.ignore_index, counter, stream);
  if (st == GH_OK && fused && cudaMemsetAsync(flags, 0, flags_bytes, stream) != cudaSuccess) st = GH_ERR_CUDA;
  if (st == GH_OK && split_count && cudaMemsetAsync(split_count, 0, count_bytes, stream) != cudaSuccess)
    st = GH_ERR_CUDA;
  // W as the K-major B operand of the logits GEMM and the N-major B operand of
  // dX; the weight-gradient output (bf16) and accumulator (fp32) maps.
  CUtensorMap tm_w_k, tm_w_n, tm_dw_out, tm_acc, tm_ws;
  if (st == GH_OK &&
      (!make_tmap(&tm_w_k, W, D, V, D * 2, pair ? sm100::GemmCfg<true>::kBRows : sm100::GemmCfg<false>::kBRows) || !make_tmap(&tm_w_n, W, D, V, D * 2, 64) ||
       (!out32 && !make_out_bf16(&tm_dw_out, dW, D, V, D)) || ((acc32 || out32) && !make_out_f32(&tm_acc, acc, D, V, D)) ||
       (ws && !make_out_f32(&tm_ws, ws, D, dx_splits * rows_pad, D))))
    st = GH_ERR_CUDA;

  int split_base = 0;  // arrivals per split counter so far in this call (cooperative split sums)
  for (int64_t c = 0; c < nchunks && st == GH_OK; ++c) {
    const int64_t c0 = c * chunk;
    const int rows = static_cast<int>(std::min<int64_t>(chunk, N - c0));
    const uint16_t* Xc = X + c0 * D;
    const int m = static_cast<int>(c % grp);     // this chunk's place in its group
    const int64_t gi = c / grp;                  // the group's index
    uint16_t* Lm = fused ? L + m * chunk * 64 : L;          // its exponentials (first row)
    uint16_t* Xsm = fused ? Xs + m * chunk * D : nullptr;  // its scaled inputs

    CUtensorMap tm_x_k, tm_l_k, tm_l_out, tm_dx_out;
    const bool maps_ok =
        make_tmap(&tm_x_k, Xc, D, rows, D * 2, sm100::kBM) && make_out_bf16(&tm_dx_out, dX + c0 * D, D, rows, D) &&
        (fused ? make_pblk(&tm_l_k, Lm, rows, nblk, blk_rows, sm100::kBM, 1) &&
                     make_pblk(&tm_l_out, Lm, rows, nblk, blk_rows, 32, 2)
               : make_tmap(&tm_l_k, L, V, rows, ld * 2, sm100::kBM) && make_out_bf16(&tm_l_out, L, V, rows, ld));
    if (!maps_ok) {
      st = GH_ERR_CUDA;
      break;
    }

    if (fused) {
      // 1: P = exp(X_c W^T) with the row statistics
      sm100::GemmArgs g1 = gemm_args(rows, static_cast<int>(V), static_cast<int>(D), 1, sm100::kEpiCeExp, pair);
      g1.targets = a.targets + c0;
      g1.ignore_index = a.ignore_index;
      g1.stats = stats;
      g1.stats_ld = static_cast<int>(rows_pad);
      g1.x_target = x_target;
      g1.out_blocked = 1;
      st = launch_gemm<false, false>(tm_x_k, tm_w_k, tm_l_out, g1, pair, GH_KERNEL_LOGITS_GEMM, stream);
      if (st != GH_OK) break;
      // 2: lse, loss, alpha, the target entries and the scaled inputs
      FinalizeArgs fa{};
      fa.stats = stats;
      fa.stats_ld = static_cast<int>(rows_pad);
      fa.tiles_n = tiles_n_logits;
      fa.targets = a.targets + c0;
      fa.ignore_index = a.ignore_index;
      fa.V = static_cast<int>(V);
      fa.rows = rows;
      fa.D = static_cast<int>(D);
      fa.z = a.z;
      fa.mean = a.mean;
      fa.n_valid = n_valid;
      fa.x_target = x_target;
      fa.row_max = row_max;
      fa.flag = flags + c;
      fa.alpha = alpha;
      fa.row_loss = row_loss + c0;
      fa.P = Lm;
      fa.blk_rows = blk_rows;
      fa.X = Xc;
      fa.Xs = Xsm;
      const dim3 fgrid(static_cast<unsigned>((rows + 31) / 32));
      {
        ProfileScope prof(GH_KERNEL_CHUNK_CE, stream);
        const cudaError_t e = launch_pdl(lce_finalize_kernel, fgrid, dim3(kFinWarps * 32), 0, stream, 1, fa);
        note_launch();
        if (e != cudaSuccess) {
          st = GH_ERR_CUDA;
          break;
        }
      }
      // 3: the recompute with R = the row max, for a chunk whose flag the finalize set
      sm100::GemmArgs g1r = g1;
      g1r.row_ref = row_max;
      g1r.run_flag = flags + c;
      st = launch_gemm<false, false>(tm_x_k, tm_w_k, tm_l_out, g1r, pair, GH_KERNEL_CHUNK_CE, stream);
      if (st != GH_OK) break;
      fa.recompute = 1;
      {
        ProfileScope prof(GH_KERNEL_CHUNK_CE, stream);
        const cudaError_t e = launch_pdl(lce_finalize_kernel, fgrid, dim3(kFinWarps * 32), 0, stream, 1, fa);
        note_launch();
        if (e != cudaSuccess) {
          st = GH_ERR_CUDA;
          break;
        }
      }
    } else {
      // 1: L = X_c W^T
      sm100::GemmArgs g1 = gemm_args(rows, static_cast<int>(V), static_cast<int>(D), 1, sm100::kEpiStoreBf16, pair);
      st = launch_gemm<false, false>(tm_x_k, tm_w_k, tm_l_out, g1, pair, GH_KERNEL_LOGITS_GEMM, stream);
      if (st != GH_OK) break;
      // 2: the caller's loss and logits gradient, in place
      st = a.loss_fn(a.loss_ctx, c0, rows, L, ld, V, a.loss, stream);
      if (st != GH_OK) break;
    }

    // 3: dX_c = G_c W (K split into fp32 partials when the tiles alone leave SMs idle)
    sm100::GemmArgs g3 = gemm_args(rows, static_cast<int>(D), static_cast<int>(V), 1, sm100::kEpiStoreBf16, pair);
    g3.row_scale = alpha;  // null on the plain path
    g3.a_blocked = fused;
    const int splits = choose_splits(g3.tiles_m * g3.tiles_n, g3.num_kb, units, sm100::kMaxSplits);
    if (splits > 1 && ws) {
      g3.k_splits = std::min(splits, dx_splits);
      g3.kb_per_split = (g3.num_kb + g3.k_splits - 1) / g3.k_splits;
      g3.k_splits = (g3.num_kb + g3.kb_per_split - 1) / g3.kb_per_split;
      g3.split_rows = static_cast<int>(rows_pad);
      g3.epi = sm100::kEpiStoreF32;
      // the last split to finish each 32-row slice sums the partials in split order
      g3.split_ws = ws;
      g3.split_out = dX + c0 * D;
      g3.split_ld = D;
      g3.split_count = split_count;
      if (g3.tiles_m * g3.tiles_n * g3.k_splits <= units) {
        // every unit has its own SM (pair) at once: the splits share the sums
        split_base += g3.k_splits;
        g3.split_target = split_base;
      }
      st = launch_gemm<false, true>(tm_l_k, tm_w_n, tm_ws, g3, pair, GH_KERNEL_DX_GEMM, stream);
      if (st != GH_OK) break;
    } else {
      st = launch_gemm<false, true>(tm_l_k, tm_w_n, tm_dx_out, g3, pair, GH_KERNEL_DX_GEMM, stream);
      if (st != GH_OK) break;
    }

    // 4: dW (+)= G^T X over the group's chunks, once its last chunk is done
    if (m + 1 < grp && c + 1 < nchunks) continue;
    const int64_t g0 = gi * grp * chunk;                                   // the group's first row
    const int grows = static_cast<int>(std::min<int64_t>(grp * chunk, N - g0));  // its rows (K)
    // the B operand of dW: the inputs, scaled by alpha on the fused path
    CUtensorMap tm_l_m, tm_x_n;
    if (!(fused ? make_pblk(&tm_l_m, L, grows, nblk, blk_rows, 64, 2) && make_tmap(&tm_x_n, Xs, D, grows, D * 2, 64)
                : make_tmap(&tm_l_m, L, V, rows, ld * 2, 64) && make_tmap(&tm_x_n, Xc, D, rows, D * 2, 64))) {
      st = GH_ERR_CUDA;
      break;
    }
    sm100::GemmArgs g4 = gemm_args(static_cast<int>(V), static_cast<int>(D), grows, 0, sm100::kEpiStoreBf16, pair);
    g4.a_blocked = fused;
    // dW reads P and the (scaled) inputs, which the dX GEMM before it waited
    // for before letting dependents launch, and nothing dX writes: its tiles
    // start as dX's CTAs retire; it completes after dX, so the next chunk's
    // logits GEMM cannot overwrite P while dW reads it.
    g4.defer_wait = 1;
    const CUtensorMap* out4 = &tm_dw_out;
    if (out32) {
      g4.epi = gi == 0 ? sm100::kEpiStoreF32 : sm100::kEpiAddF32;
      out4 = &tm_acc;
    } else if (a.accum == GH_ACCUM_FP32) {
      if (acc32 && gi + 1 < ngroups) {
        g4.epi = gi == 0 ? sm100::kEpiStoreF32 : sm100::kEpiAddF32;
        out4 = &tm_acc;
      } else if (acc32) {
        // the last group adds its product to the fp32 accumulator and rounds
        // the sum to bf16 once, straight into grad_weight
        g4.epi = sm100::kEpiAccToBf16;
      }
    } else {
      g4.epi = c == 0 ? sm100::kEpiStoreBf16 : sm100::kEpiBf16Add;
    }
    if (out32 && a.on_slice && c + 1 == nchunks && fused) {
      // the last contraction in ranges of weight rows (whole tiles), each
      // handed to the caller once enqueued
      const int tiles_all = g4.tiles_m;
      const int slices = static_cast<int>(std::min<int64_t>(std::max<int64_t>(a.dw_slices, 1), tiles_all));
      for (int s = 0; s < slices && st == GH_OK; ++s) {
        const int64_t v0 = static_cast<int64_t>(tiles_all) * s / slices * tile_m;
        const int64_t v1 = std::min<int64_t>(V, static_cast<int64_t>(tiles_all) * (s + 1) / slices * tile_m);
        CUtensorMap tm_a_s, tm_o_s;
        if (!make_pblk(&tm_a_s, L + (v0 / 64) * blk_rows * 64, grows, (v1 - v0 + 63) / 64, blk_rows, 64, 2) ||
            !make_out_f32(&tm_o_s, acc + v0 * D, D, v1 - v0, D)) {
          st = GH_ERR_CUDA;
          break;
        }
        sm100::GemmArgs gs = gemm_args(static_cast<int>(v1 - v0), static_cast<int>(D), grows, 0, g4.epi, pair);
        gs.a_blocked = 1;
        gs.defer_wait = 1;
        st = launch_gemm<true, true>(tm_a_s, tm_x_n, tm_o_s, gs, pair, GH_KERNEL_DW_GEMM, stream, nullptr,
                                     a.max_sms);
        if (st == GH_OK) st = a.on_slice(a.slice_ctx, v0, v1, stream);
      }
    } else {
      st = launch_gemm<true, true>(tm_l_m, tm_x_n, *out4, g4, pair, GH_KERNEL_DW_GEMM, stream,
                                   g4.epi == sm100::kEpiAccToBf16 ? &tm_acc : nullptr);
    }
  }
  if (st == GH_OK && !custom) st = ce_reduce_launch(row_loss, N, n_valid, a.mean, a.loss, stream);
  scratch_free(scratch, stream);
  return st;
}

}  // namespace gh
