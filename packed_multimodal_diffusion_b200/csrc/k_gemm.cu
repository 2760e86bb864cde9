// Host launchers of the tcgen05 GEMM instantiations and the TMA tensor-map
// encoder.  The block's four projections ("cortiq_engine/mmh3.rs",
// block_forward / ffn_tail: qkv, out, fc1, fc2), the output heads and the
// patch / condition projections of forward and refine_text, and the encoder
// layer's four biased projections ("ffai-argus 0.7.0 src/siglip.rs",
// Layer::forward / finish_attention) all go through gemm_tc_kernel or its
// CTA-pair form gemm2_tc_kernel with the matching fused epilogue.  Which one
// runs is fixed per call shape (use_pairs and the dispatch below), not
// switched at run time.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdlib>
#include <mutex>

#include "gemm_tc.cuh"
#include "mmh3_internal.h"

namespace mmh3 {

// ----------------------------------------------------------- tensor maps
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool make_tmap_2d(CUtensorMap* m, const void* base, int esize, uint64_t cols, uint64_t rows,
                  uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * (uint64_t)esize};
  const cuuint32_t box[2] = {(cuuint32_t)(128 / esize), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt = esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- launch
// Row tiles per group of the persistent tile order (see tile_coords).  A
// group's A panel (group_m row tiles x K) is reused by every column tile of
// the group, and B is swept once per group; the L2 that a working set can
// count on is about one die's half (whole-operand residency of 58-71 MB
// thrashed: A or B re-read 6-12 times), so the panel is kept to about
// 24 MB.  With few column tiles (N <= 16 tiles) a group of at most 8 row
// tiles measured best (the out and fc2 GEMMs of the block workload).
// Measured at that workload, group sizes 1..52, two alternating rounds:
// qkv 0.42 ms for 8..26, fc1 0.943-0.955 ms at 26 (1.06 at 1), fc2 0.53 ms
// for 1..16 (0.62 at 52), out 0.147-0.150 ms for 2..8.  MMH3_GEMM_GROUP_M=<g>
// (g >= 1) overrides the choice, for such measurements.
static int group_m_for(int K, int n_tiles, int m_tiles, int bm) {
  static int forced = -1;
  if (forced < 0) {
    const char* v = std::getenv("MMH3_GEMM_GROUP_M");
    forced = v ? std::max(0, std::atoi(v)) : 0;
  }
  if (forced > 0) return std::min(forced, m_tiles);
  const int64_t row_tile_bytes = (int64_t)bm * K * 2;
  int g = (int)std::max<int64_t>(1, ((int64_t)24 << 20) / row_tile_bytes);
  if (n_tiles <= 16) g = std::min(g, 8);
  return std::min(g, m_tiles);
}

template <int BN, int OUT>
constexpr int stages_for() {
  constexpr int base = BN >= 256 ? 4 : (BN >= 224 ? 5 : 6);
  constexpr int fit = (232448 - OUT - 1024 - 256 - kEpiSmemBytes) / GemmShape<BN>::kStageBytes;
  return base < fit ? base : fit;
}

// out / out_esize / out_cols: the [M, out_cols] tensor a staged epilogue
// loads and stores with TMA (bf16 or fp32).
template <typename T, int BN, class Epi>
static mmh3_status run_gemm(const void* A, const void* B, int M, int N, int K, const Epi& epi,
                            cudaStream_t s, const void* out = nullptr, int out_esize = 0, int out_cols = 0) {
  constexpr int OUT = Epi::kStageOut;
  constexpr int STAGES = stages_for<BN, OUT>();
  constexpr int smem = gemm_smem_bytes<BN, STAGES, OUT>();
  static_assert(STAGES >= 4, "GEMM: fewer than four operand stages fit");
  static_assert(smem <= 232448, "GEMM shared memory above the per-CTA limit");
  if (M <= 0) return MMH3_OK;
  if (fault_injected("tensormap")) return fail(MMH3_ERR_CUDA, "injected fault at tensormap");
  const int es = (int)sizeof(T);
  if ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(B) | reinterpret_cast<uintptr_t>(out)) & 15)
    return fail(MMH3_ERR_ALIGN, "GEMM operand not 16-byte aligned");
  if (((size_t)K * es) % 16 != 0) return fail(MMH3_ERR_SHAPE, "GEMM K=%d row pitch not a multiple of 16 bytes", K);
  CUtensorMap ta, tb, tc;
  if (!make_tmap_2d(&ta, A, es, (uint64_t)K, (uint64_t)M, 128) ||
      !make_tmap_2d(&tb, B, es, (uint64_t)K, (uint64_t)N, BN))
    return fail(MMH3_ERR_CUDA, "cuTensorMapEncodeTiled failed (M=%d N=%d K=%d)", M, N, K);
  if constexpr (OUT > 0) {
    if (out == nullptr || (out_cols * out_esize) % 128 != 0)
      return fail(MMH3_ERR_SHAPE, "staged epilogue: output row of %d x %d bytes not a multiple of 128", out_cols,
                  out_esize);
    if (!make_tmap_2d(&tc, out, out_esize, (uint64_t)out_cols, (uint64_t)M, 128))
      return fail(MMH3_ERR_CUDA, "cuTensorMapEncodeTiled failed for the output (M=%d, %d columns)", M, out_cols);
  } else {
    tc = ta;  // not read
  }
  auto kern = gemm_tc_kernel<T, BN, STAGES, Epi>;
  {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "GEMM smem attribute");
  }
  const int m_tiles = (M + 127) / 128;
  const int tiles = m_tiles * ((N + BN - 1) / BN);
  const int grid = tiles < num_sms() ? tiles : num_sms();
  if (fault_injected("launch")) return fail(MMH3_ERR_CUDA, "injected fault at launch");
  const int gm = group_m_for(K, (N + BN - 1) / BN, m_tiles, 128);
  cudaError_t e = launch_pdl(kern, dim3(grid), dim3(kGemmThreads), smem, s, ta, tb, tc, M, N, K, gm, epi,
                             device_status_ptr(), wait_limit_ns());
  count_launch();
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "GEMM launch");
  return MMH3_OK;
}

// ---------------------------------------------------- CTA-pair launch
// As many operand stages as fit beside the output staging and the
// epilogue's parameters (at most 8).
template <int BN, class Epi>
constexpr int stages2_for() {
  constexpr int fixed = Epi::kStageOut + 1024 + 256 + ((Epi::kSmemFloats * 4 + 255) / 256) * 256;
  constexpr int n = (232448 - fixed) / Gemm2Shape<BN>::kStageBytes;
  return n > 8 ? 8 : n;
}

// out / out_cols / out_esize: the [M, out_cols] tensor (bf16 or fp32) a
// staged epilogue loads and stores with TMA.
template <int BN, class Epi>
static mmh3_status run_gemm2(const void* A, const void* B, int M, int N, int K, const Epi& epi,
                             cudaStream_t s, const void* out = nullptr, int out_cols = 0, int out_esize = 2) {
  constexpr int STAGES = stages2_for<BN, Epi>();
  constexpr int smem = gemm2_smem_bytes<BN, STAGES, Epi>();
  static_assert(STAGES >= 4, "pair GEMM: fewer than four operand stages fit");
  static_assert(smem <= 232448, "pair GEMM shared memory above the per-CTA limit");
  if (M <= 0) return MMH3_OK;
  if (fault_injected("tensormap")) return fail(MMH3_ERR_CUDA, "injected fault at tensormap");
  if ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(B) | reinterpret_cast<uintptr_t>(out)) & 15)
    return fail(MMH3_ERR_ALIGN, "GEMM operand not 16-byte aligned");
  if (((size_t)K * 2) % 16 != 0) return fail(MMH3_ERR_SHAPE, "GEMM K=%d row pitch not a multiple of 16 bytes", K);
  CUtensorMap ta, tb, tc;
  if (!make_tmap_2d(&ta, A, 2, (uint64_t)K, (uint64_t)M, 128) ||
      !make_tmap_2d(&tb, B, 2, (uint64_t)K, (uint64_t)N, BN / 2))
    return fail(MMH3_ERR_CUDA, "cuTensorMapEncodeTiled failed (M=%d N=%d K=%d)", M, N, K);
  if constexpr (Epi::kStageOut > 0) {
    if (out == nullptr || (out_cols * out_esize) % 128 != 0)
      return fail(MMH3_ERR_SHAPE, "staged epilogue: output row of %d x %d bytes not a multiple of 128", out_cols,
                  out_esize);
    if (!make_tmap_2d(&tc, out, out_esize, (uint64_t)out_cols, (uint64_t)M, 128))
      return fail(MMH3_ERR_CUDA, "cuTensorMapEncodeTiled failed for the output (M=%d, %d columns)", M, out_cols);
  } else {
    tc = ta;  // not read
  }
  auto kern = gemm2_tc_kernel<BN, STAGES, Epi>;
  static int max_pairs = -1;  // per instantiation, from the occupancy query
  if (max_pairs < 0) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "pair GEMM smem attribute");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * num_sms(), 1, 1);
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
    if (e != cudaSuccess) return cuda_fail(e, "pair GEMM occupancy query");
    if (n < 1) return fail(MMH3_ERR_CUDA, "pair GEMM: no CTA pair fits on this device");
    max_pairs = n;
  }
  const int m_tiles = (M + 255) / 256;
  const int tiles = m_tiles * ((N + BN - 1) / BN);
  const int pairs = tiles < max_pairs ? tiles : max_pairs;
  if (fault_injected("launch")) return fail(MMH3_ERR_CUDA, "injected fault at launch");
  const int gm = group_m_for(K, (N + BN - 1) / BN, m_tiles, 256);
  cudaError_t e = launch_pdl(kern, dim3(2 * pairs), dim3(kGemmThreads), smem, s, ta, tb, tc, M, N, K, gm, epi,
                             device_status_ptr(), wait_limit_ns());
  count_launch();
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pair GEMM launch");
  return MMH3_OK;
}

// The pair kernel serves bf16 GEMMs with at least one full pair of row
// tiles.  Each CTA's half of the last column tile lies wholly inside or
// wholly beyond N (a load beyond N reads zeros; the epilogue skips it).
static bool use_pairs(int M, int N, int BN) { return M >= 256 && N % (BN / 2) == 0; }

// qkv + per-head RMSNorm + rotation
mmh3_status gemm_qkv(int dtype, const void* A, const void* B, int M, int N, int K, int head_dim,
                     int inner, const float* q_norm, const float* k_norm, const float2* cs,
                     float eps, void* out, cudaStream_t s) {
  if (dtype == MMH3_BF16 && head_dim == 128) {
    if (use_pairs(M, N, 256)) {
      EpiQkvNormRopeTma<256> e{N, inner, q_norm, k_norm, cs, M, eps};
      return run_gemm2<256>(A, B, M, N, K, e, s, out, N);
    }
    EpiQkvNormRope<__nv_bfloat16, 128, 256> e{static_cast<__nv_bfloat16*>(out), N, inner, q_norm, k_norm, cs, M, eps};
    return run_gemm<__nv_bfloat16, 256>(A, B, M, N, K, e, s);
  }
  if (dtype == MMH3_BF16 && head_dim == 64) {
    EpiQkvNormRope<__nv_bfloat16, 64, 256> e{static_cast<__nv_bfloat16*>(out), N, inner, q_norm, k_norm, cs, M, eps};
    return run_gemm<__nv_bfloat16, 256>(A, B, M, N, K, e, s);
  }
  if (dtype == MMH3_F32 && head_dim == 64) {
    EpiQkvNormRope<float, 64, 256> e{static_cast<float*>(out), N, inner, q_norm, k_norm, cs, M, eps};
    return run_gemm<float, 256>(A, B, M, N, K, e, s);
  }
  if (dtype == MMH3_F32 && head_dim == 128) {
    EpiQkvNormRope<float, 128, 256> e{static_cast<float*>(out), N, inner, q_norm, k_norm, cs, M, eps};
    return run_gemm<float, 256>(A, B, M, N, K, e, s);
  }
  return fail(MMH3_ERR_SHAPE, "qkv: head_dim %d unsupported", head_dim);
}

mmh3_status gemm_gated_residual(int dtype, const void* A, const void* B, int M, int N, int K,
                                float* x, const float* mods, int mods_stride, int chunk_off,
                                const SegRows& seg, cudaStream_t s) {
  if (dtype == MMH3_BF16) {
    // CTA pairs with 256-wide tiles for the out projection and for fc2
    // (K = 4H), even where N leaves the last column tile half empty (N =
    // 2688: 10.5 tiles).  Per SM and 64-deep k-block a 256 x 192 pair tile
    // moves 28 KB through shared memory twice (TMA in, MMA out) in 384 MMA
    // cycles, about 146 B/clk against the 128 B/clk shared memory gives; a
    // 256 x 256 tile needs 125.  Measured in the same calls: fc2 0.540-0.545
    // against 0.550-0.553 ms with 192-wide tiles, out unchanged.  When N is a
    // multiple of 32 the update is added into x by tensor reduce-adds.
    const bool staged = N % 32 == 0;
    if (staged && use_pairs(M, N, 256)) {
      EpiResidualTma<256, false> e{{}, N, mods, mods_stride, chunk_off, seg, nullptr};
      return run_gemm2<256>(A, B, M, N, K, e, s, x, N, 4);
    }
    if (staged && N % 192 == 0 && use_pairs(M, N, 192)) {
      EpiResidualTma<192, false> e{{}, N, mods, mods_stride, chunk_off, seg, nullptr};
      return run_gemm2<192>(A, B, M, N, K, e, s, x, N, 4);
    }
    if (staged && N % 224 == 0) {
      EpiResidualTma<224, false> e{{}, N, mods, mods_stride, chunk_off, seg, nullptr};
      return run_gemm<__nv_bfloat16, 224>(A, B, M, N, K, e, s, x, 4, N);
    }
    if (N % 256 == 0) {
      EpiGatedResidual<256> e{{}, x, N, mods, mods_stride, chunk_off, seg, nullptr};
      return run_gemm<__nv_bfloat16, 256>(A, B, M, N, K, e, s);
    }
    if (N % 224 == 0) {
      EpiGatedResidual<224> e{{}, x, N, mods, mods_stride, chunk_off, seg, nullptr};
      return run_gemm<__nv_bfloat16, 224>(A, B, M, N, K, e, s);
    }
    EpiGatedResidual<128> e{{}, x, N, mods, mods_stride, chunk_off, seg, nullptr};
    return run_gemm<__nv_bfloat16, 128>(A, B, M, N, K, e, s);
  }
  if (N % 256 == 0) {
    EpiGatedResidual<256> e{{}, x, N, mods, mods_stride, chunk_off, seg, nullptr};
    return run_gemm<float, 256>(A, B, M, N, K, e, s);
  }
  EpiGatedResidual<128> e{{}, x, N, mods, mods_stride, chunk_off, seg, nullptr};
  return run_gemm<float, 128>(A, B, M, N, K, e, s);
}

mmh3_status gemm_swiglu(int dtype, const void* A, const void* B, int M, int F, int K, void* out,
                        cudaStream_t s) {
  if (dtype == MMH3_BF16) {
    if (use_pairs(M, 2 * F, 256) && F % 64 == 0) {
      EpiSwiGLUTma<256> et{{}, F};
      return run_gemm2<256>(A, B, M, 2 * F, K, et, s, out, F);
    }
    EpiSwiGLU<__nv_bfloat16, 256> e{{}, static_cast<__nv_bfloat16*>(out), F};
    return run_gemm<__nv_bfloat16, 256>(A, B, M, 2 * F, K, e, s);
  }
  EpiSwiGLU<float, 256> e{{}, static_cast<float*>(out), F};
  return run_gemm<float, 256>(A, B, M, 2 * F, K, e, s);
}

mmh3_status gemm_bias_act(int dtype, const void* A, const void* B, int M, int N, int K,
                          const float* bias, int mode, void* out, cudaStream_t s) {
  if (mode == 3) {  // fp32 output with bias (patch and condition projections)
    if (dtype == MMH3_BF16) {
      EpiBiasAct<float, 256, 0> e{{}, static_cast<float*>(out), N, bias};
      return run_gemm<__nv_bfloat16, 256>(A, B, M, N, K, e, s);
    }
    EpiBiasAct<float, 256, 0> e{{}, static_cast<float*>(out), N, bias};
    return run_gemm<float, 256>(A, B, M, N, K, e, s);
  }
  if (mode == 2) {  // output heads: fp32, negated, N = 128-wide tiles
    if (dtype == MMH3_BF16) {
      EpiBiasAct<float, 128, 2> e{{}, static_cast<float*>(out), N, bias};
      return run_gemm<__nv_bfloat16, 128>(A, B, M, N, K, e, s);
    }
    EpiBiasAct<float, 128, 2> e{{}, static_cast<float*>(out), N, bias};
    return run_gemm<float, 128>(A, B, M, N, K, e, s);
  }
  if (dtype != MMH3_BF16) return fail(MMH3_ERR_UNSUPPORTED, "bias/gelu epilogue: bf16 only");
  // the pair kernel's epilogue reads the bias as float4
  const bool bias16 = (reinterpret_cast<uintptr_t>(bias) & 15) == 0;
  if (mode == 1) {
    if (use_pairs(M, N, 256) && N % 64 == 0 && bias16) {
      EpiBiasActTma<256, 1> et{{}, N, bias};
      return run_gemm2<256>(A, B, M, N, K, et, s, out, N);
    }
    EpiBiasAct<__nv_bfloat16, 256, 1> e{{}, static_cast<__nv_bfloat16*>(out), N, bias};
    return run_gemm<__nv_bfloat16, 256>(A, B, M, N, K, e, s);
  }
  if (use_pairs(M, N, 256) && N % 64 == 0 && bias16) {
    EpiBiasActTma<256, 0> et{{}, N, bias};
    return run_gemm2<256>(A, B, M, N, K, et, s, out, N);
  }
  EpiBiasAct<__nv_bfloat16, 256, 0> e{{}, static_cast<__nv_bfloat16*>(out), N, bias};
  return run_gemm<__nv_bfloat16, 256>(A, B, M, N, K, e, s);
}

mmh3_status gemm_bias_residual(int dtype, const void* A, const void* B, int M, int N, int K,
                               const float* bias, float* x, cudaStream_t s) {
  if (dtype != MMH3_BF16) return fail(MMH3_ERR_UNSUPPORTED, "bias residual epilogue: bf16 only");
  if ((reinterpret_cast<uintptr_t>(bias) & 15) != 0)  // both epilogues read it as float4
    return fail(MMH3_ERR_ALIGN, "bias residual epilogue: bias not 16-byte aligned");
  if (use_pairs(M, N, 256) && N % 32 == 0) {
    EpiResidualTma<256, true> et{{}, N, nullptr, 0, 0, SegRows{}, bias};
    return run_gemm2<256>(A, B, M, N, K, et, s, x, N, 4);
  }
  EpiBiasResidual<256> e{{}, x, N, nullptr, 0, 0, SegRows{}, bias};
  return run_gemm<__nv_bfloat16, 256>(A, B, M, N, K, e, s);
}

}  // namespace mmh3
