// Chunked linear cross-entropy (Greyhound `chunked_linear_cross_entropy` over
// `chunked_linear_loss`): logits = X @ W^T are formed one row chunk at a time
// and never materialised in full.  Per chunk c (rows [c0, c0 + rows)):
//
//   1  L      = X_c W^T               tcgen05 GEMM, bf16 chunk buffer [rows, ld]
//   2  L     := G_c (in place)        the cross-entropy row kernel on the chunk:
//                                     loss rows and the logits gradient, scaled
//                                     by the valid-token count of the whole call
//   3  dX_c   = G_c W                 tcgen05 GEMM (A K-major, B N-major)
//   4  dW    (+)= G_c^T X_c           tcgen05 GEMM (both operands M/N-major);
//                                     fp32 accumulator across chunks, cast once
//                                     by the last chunk's epilogue ("fp32"), or
//                                     accumulated in the bf16 output ("weight")
//
// The loss is the fixed-order sum of all rows' losses, divided by the valid
// count for "mean".  ld = round_up(V, 8) keeps chunk rows 16-byte aligned as
// TMA requires; TMA reads the chunk with extent V, so its padding columns are
// never used.
#include <algorithm>
#include <cstdlib>
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

// 2-D bf16 tensor map: `inner` contiguous elements per row, `outer` rows of
// `row_bytes`, box {64, box_outer}, 128-byte swizzle, zero fill outside.
bool make_tmap(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
               uint32_t box_outer) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {64, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

template <bool A_MN, bool B_MN>
gh_status_t launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const sm100::GemmArgs& g, int kind,
                        cudaStream_t stream) {
  auto kern = sm100::gemm_bf16_kernel<A_MN, B_MN>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, sm100::kGemmSmem);
  });
  if (attr_err != cudaSuccess) return GH_ERR_CUDA;
  const int tiles = g.tiles_m * g.tiles_n;
  if (tiles == 0) return GH_OK;
  const int grid = std::min(tiles, sm_count());
  ProfileScope prof(kind, stream);
  kern<<<grid, sm100::kGemmThreads, sm100::kGemmSmem, stream>>>(ta, tb, g);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? GH_OK : GH_ERR_CUDA;
}

int64_t default_chunk(int64_t N, int64_t ld) {
  // Largest multiple of 128 rows whose bf16 chunk logits fit in 1 GiB, capped at N.
  int64_t c = ((int64_t(1) << 30) / (ld * 2)) / 128 * 128;
  c = std::max<int64_t>(c, 128);
  return std::min<int64_t>(c, std::max<int64_t>(N, 1));
}

}  // namespace

gh_status_t linear_ce_run(const LinearCeArgs& a, cudaStream_t stream) {
  const int64_t N = a.N, D = a.D, V = a.V;
  if (N == 0) {
    // No token: zero loss, zero weight gradient.
    if (cudaMemsetAsync(a.loss, 0, sizeof(float), stream) != cudaSuccess) return GH_ERR_CUDA;
    if (cudaMemsetAsync(a.dW, 0, static_cast<size_t>(V) * D * 2, stream) != cudaSuccess) return GH_ERR_CUDA;
    return GH_OK;
  }
  if (!tensor_map_encoder()) return GH_ERR_UNSUPPORTED;
  const int64_t ld = (V + 7) / 8 * 8;
  int64_t chunk = a.chunk > 0 ? std::min<int64_t>(a.chunk, N) : default_chunk(N, ld);
  const int64_t nchunks = (N + chunk - 1) / chunk;
  if (chunk > INT32_MAX / 2 || V > INT32_MAX / 2) return GH_ERR_UNSUPPORTED;
  const bool acc32 = a.accum == GH_ACCUM_FP32 && nchunks > 1;

  // scratch: [counter | row losses | chunk buffer | fp32 accumulator]
  const size_t off_rows = 256;
  const size_t off_buf = (off_rows + sizeof(float) * N + 255) / 256 * 256;
  const size_t buf_bytes = static_cast<size_t>(chunk) * ld * 2;
  const size_t off_acc = (off_buf + buf_bytes + 255) / 256 * 256;
  const size_t total = off_acc + (acc32 ? static_cast<size_t>(V) * D * 4 : 0);
  void* scratch = nullptr;
  gh_status_t st = scratch_alloc(&scratch, total, stream);
  if (st != GH_OK) return st;
  char* base = static_cast<char*>(scratch);
  unsigned long long* n_valid = reinterpret_cast<unsigned long long*>(base);
  float* row_loss = reinterpret_cast<float*>(base + off_rows);
  uint16_t* L = reinterpret_cast<uint16_t*>(base + off_buf);
  float* acc = acc32 ? reinterpret_cast<float*>(base + off_acc) : nullptr;

  const uint16_t* X = static_cast<const uint16_t*>(a.X);
  const uint16_t* W = static_cast<const uint16_t*>(a.W);
  uint16_t* dX = static_cast<uint16_t*>(a.dX);
  uint16_t* dW = static_cast<uint16_t*>(a.dW);

  st = ce_count_launch(a.targets, N, V, a.ignore_index, n_valid, stream);
  // W as the K-major B operand of the logits GEMM and the N-major B operand of dX.
  CUtensorMap tm_w_k, tm_w_n;
  if (st == GH_OK && (!make_tmap(&tm_w_k, W, D, V, D * 2, sm100::kBN) || !make_tmap(&tm_w_n, W, D, V, D * 2, 64)))
    st = GH_ERR_CUDA;

  for (int64_t c = 0; c < nchunks && st == GH_OK; ++c) {
    const int64_t c0 = c * chunk;
    const int rows = static_cast<int>(std::min<int64_t>(chunk, N - c0));
    const uint16_t* Xc = X + c0 * D;

    // 1: L = X_c W^T
    CUtensorMap tm_x_k, tm_l_k, tm_l_m, tm_x_n;
    if (!make_tmap(&tm_x_k, Xc, D, rows, D * 2, sm100::kBM) || !make_tmap(&tm_l_k, L, V, rows, ld * 2, sm100::kBM) ||
        !make_tmap(&tm_l_m, L, V, rows, ld * 2, 64) || !make_tmap(&tm_x_n, Xc, D, rows, D * 2, 64)) {
      st = GH_ERR_CUDA;
      break;
    }
    sm100::GemmArgs g1{};
    g1.M = rows; g1.N = static_cast<int>(V); g1.K = static_cast<int>(D);
    g1.tiles_m = (rows + sm100::kBM - 1) / sm100::kBM;
    g1.tiles_n = static_cast<int>((V + sm100::kBN - 1) / sm100::kBN);
    g1.num_kb = static_cast<int>((D + sm100::kBK - 1) / sm100::kBK);
    g1.m_fastest = 1;
    g1.epi = sm100::kEpiStoreBf16;
    g1.out = L; g1.ld_out = ld;
    g1.m_limit = rows; g1.n_limit = static_cast<int>(ld);
    st = launch_gemm<false, false>(tm_x_k, tm_w_k, g1, GH_KERNEL_LOGITS_GEMM, stream);
    if (st != GH_OK) break;

    // 2: per-row loss and the logits gradient, in place
    CeArgs ca{};
    ca.logits = L;
    ca.grad = L;
    ca.targets = a.targets + c0;
    ca.V = V;
    ca.ld = ld;
    ca.ignore_index = a.ignore_index;
    ca.z = a.z;
    ca.mean = a.mean;
    ca.n_valid = n_valid;
    ca.row_loss = row_loss + c0;
    ca.congruent = 1;
    ca.profile_kind = GH_KERNEL_CHUNK_CE;
    st = ce_launch(ca, rows, GH_BF16, stream);
    if (st != GH_OK) break;

    // 3: dX_c = G_c W
    sm100::GemmArgs g3{};
    g3.M = rows; g3.N = static_cast<int>(D); g3.K = static_cast<int>(V);
    g3.tiles_m = (rows + sm100::kBM - 1) / sm100::kBM;
    g3.tiles_n = static_cast<int>((D + sm100::kBN - 1) / sm100::kBN);
    g3.num_kb = static_cast<int>((V + sm100::kBK - 1) / sm100::kBK);
    g3.m_fastest = 1;
    g3.epi = sm100::kEpiStoreBf16;
    g3.out = dX + c0 * D; g3.ld_out = D;
    g3.m_limit = rows; g3.n_limit = static_cast<int>(D);
    st = launch_gemm<false, true>(tm_l_k, tm_w_n, g3, GH_KERNEL_DX_GEMM, stream);
    if (st != GH_OK) break;

    // 4: dW (+)= G_c^T X_c
    sm100::GemmArgs g4{};
    g4.M = static_cast<int>(V); g4.N = static_cast<int>(D); g4.K = rows;
    g4.tiles_m = static_cast<int>((V + sm100::kBM - 1) / sm100::kBM);
    g4.tiles_n = static_cast<int>((D + sm100::kBN - 1) / sm100::kBN);
    g4.num_kb = (rows + sm100::kBK - 1) / sm100::kBK;
    g4.m_fastest = 0;
    g4.out = dW; g4.ld_out = D;
    g4.acc = acc; g4.ld_acc = D;
    g4.m_limit = static_cast<int>(V); g4.n_limit = static_cast<int>(D);
    if (a.accum == GH_ACCUM_FP32) {
      if (nchunks == 1) g4.epi = sm100::kEpiStoreBf16;
      else if (c == 0) g4.epi = sm100::kEpiAccWrite;
      else if (c + 1 < nchunks) g4.epi = sm100::kEpiAccAdd;
      else g4.epi = sm100::kEpiAccFinal;
    } else {
      g4.epi = c == 0 ? sm100::kEpiStoreBf16 : sm100::kEpiBf16Add;
    }
    st = launch_gemm<true, true>(tm_l_m, tm_x_n, g4, GH_KERNEL_DW_GEMM, stream);
  }
  if (st == GH_OK) st = ce_reduce_launch(row_loss, N, n_valid, a.mean, a.loss, stream);
  scratch_free(scratch, stream);
  return st;
}

}  // namespace gh
