// Internal host-side interfaces shared by the library's translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mmh3.h"
#include "mmh3_types.h"

struct CUtensorMap_st;
typedef struct CUtensorMap_st CUtensorMap;

namespace mmh3 {

// ---------------------------------------------------------------- errors
mmh3_status fail(mmh3_status code, const char* fmt, ...);
void clear_error();
// MMH3_FAULT=<site>: the host planner fails at the named site (host-side
// fault injection for tests; nothing is launched).
bool fault_injected(const char* site);
mmh3_status cuda_fail(cudaError_t e, const char* what);
uint64_t wait_limit_ns();
// MMH3_CHECK mode (MMH3_CHECK=1 in the environment, or mmh3_set_check):
// device bounds checks and workspace canaries.
bool check_mode();

// Workspace canaries of the check mode: kCanaryBytes after each region.
constexpr int kCanaryBytes = 256;
constexpr int kMaxCanaries = 16;
struct CanaryList {
  uint32_t* p[kMaxCanaries];
  int n;
};
// fill (verify = false) or verify the canaries; kernel_id names the kernel
// that ran just before a verify (MMH3_PROF_K_*, 8 for the output heads)
cudaError_t launch_canary(const CanaryList& l, bool verify, int kernel_id, cudaStream_t s);
// Address of the device status word on the current device.
DevStatus* device_status_ptr();

// Launch with programmatic stream serialization (see pdl_wait): the kernel
// must call pdl_wait() before its first global memory access.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}
int num_sms();

// ------------------------------------------------------------------ plan
// Clocks of a segment: 0 the video flow clock, 1 the audio flow clock,
// 2 the visual condition clock (keyframe and reference-image rows), 3 the
// audio condition clock (reference audio rows).
constexpr int kClocks = 4;
struct Plan {
  int n_ts = 0;
  double ts[kClocks] = {0, 0, 0, 0};
  int slot[kClocks] = {-1, -1, -1, -1};  // slot of each clock (-1: unused)
  SegRows block_rows{};      // per segment: slot*3 + tag
  SegRows final_rows{};      // per segment: slot
  int seg_tag[kMaxSeg]{};
};
mmh3_status make_plan(const mmh3_segment* segs, int n_seg, int n, double sigma_v, double sigma_a,
                      Plan* p);
// Interpolation coordinates of timestep t on a table of `grid` rows.
void curve_coords(double t, int grid, int* i0, float* f);

// -------------------------------------------------------------- launches
cudaError_t launch_adaln(const float* w, const float* b, const float* table, int rank, int grid,
                         int rows_per_slot, const Plan& plan, float* out, cudaStream_t s);
// The adaLN bases of up to kAdalnBatch blocks for one prologue launch.
constexpr int kAdalnBatch = 64;
struct AdalnBatch {
  const float* w[kAdalnBatch];
  const float* b[kAdalnBatch];
  const float* table[kAdalnBatch];
};
// One launch: the modulation of ab's first n_ab blocks (block i's rows at
// mods + i * mods_stride floats) and, if pos != null, the rotation (cos,
// sin) table of n rows with k frequencies per axis.
cudaError_t launch_prologue(const AdalnBatch& ab, int n_ab, int rank, int grid, int rows_per_slot,
                            const Plan& plan, float* mods, long long mods_stride, const float* pos, int n,
                            int k, float theta, float2* cs, cudaStream_t s);
// zero_word (optional): a 4-byte word the launch sets to 0 (the attention
// ticket counter of the same call, ready before the attention launch reads
// it, since every launch in between waits for its predecessor)
cudaError_t launch_norm_mod(int dtype, const float* x, int n, int H, const float* g, float eps,
                            const float* mods, int mods_stride, int shift_off, int scale_off,
                            const SegRows& seg, int row_base, void* out, cudaStream_t s,
                            unsigned* zero_word = nullptr);
cudaError_t launch_layernorm(const float* x, int n, int H, const float* g, const float* b,
                             float eps, __nv_bfloat16* out, cudaStream_t s, unsigned* zero_word = nullptr);
cudaError_t launch_rows(const SegRows& seg, int n, int32_t* rows, cudaStream_t s);
cudaError_t launch_fc1_tile(int esize, const void* in, void* out, int F, int H, cudaStream_t s);
cudaError_t launch_vit_fold(const void* wq, const void* wk, const void* wv, const float* bq,
                            const float* bk, const float* bv, float scale, int H, void* wqkv,
                            float* bqkv, cudaStream_t s);
cudaError_t launch_selftest_wait(uint64_t limit_ns, cudaStream_t s);
// Every kernel launch the library makes is counted (mmh3_launch_count).
void count_launch();
cudaError_t launch_patchify(int dtype, const float* x, int C, int T, int H, int W, void* rows, cudaStream_t s);
cudaError_t launch_unpatchify(const float* rows, int C, int T, int H, int W, float* x, cudaStream_t s);
cudaError_t launch_pack_audio(int dtype, const float* x, int C, int T, void* rows, cudaStream_t s);
cudaError_t launch_unpack_audio(const float* rows, int C, int T, float* x, cudaStream_t s);

// ------------------------------------------------------------------ GEMMs
// C = A[M,K] B[N,K]^T with a fused epilogue; dtype = mmh3_dtype of A and B.
mmh3_status gemm_qkv(int dtype, const void* A, const void* B, int M, int N, int K, int head_dim,
                     int inner, const float* q_norm, const float* k_norm, const float2* cs,
                     float eps, void* out, cudaStream_t s);
mmh3_status gemm_gated_residual(int dtype, const void* A, const void* B, int M, int N, int K,
                                float* x, const float* mods, int mods_stride, int chunk_off,
                                const SegRows& seg, cudaStream_t s);
mmh3_status gemm_swiglu(int dtype, const void* A, const void* B, int M, int F, int K, void* out,
                        cudaStream_t s);
// mode 0: out(act dtype) = acc + bias; 1: gelu_tanh(acc + bias);
// 2: out(fp32) = -(acc + bias); 3: out(fp32) = acc + bias
mmh3_status gemm_bias_act(int dtype, const void* A, const void* B, int M, int N, int K,
                          const float* bias, int mode, void* out, cudaStream_t s);
mmh3_status gemm_bias_residual(int dtype, const void* A, const void* B, int M, int N, int K,
                               const float* bias, float* x, cudaStream_t s);
// scratch: room for the split tail's partial results; ticket: the work
// counter of a persistent launch, already zeroed on the stream (null: the
// first 256 bytes of scratch serve, zeroed by a memset; without scratch the
// launch is one CTA per work item).
mmh3_status attention(int dtype, const void* qkv, int n_seq, int seq, int heads, int head_dim,
                      float scale, void* out, cudaStream_t s, void* scratch = nullptr,
                      size_t scratch_bytes = 0, unsigned* ticket = nullptr);
mmh3_status attention_kv(int dtype, const void* q_panel, int n_q, const void* kv, int n_kv, int heads,
                         int head_dim, float scale, void* out, cudaStream_t s, void* scratch = nullptr,
                         size_t scratch_bytes = 0, unsigned* ticket = nullptr);

// The block on a caller-provided scratch region (see mmh3_workspace_size);
// mods_or_null: the caller's modulation [T_s*3, 6H] fp32 (device) in place
// of the adaLN evaluation; profile = false records no phase-profile events.
mmh3_status block_forward_impl(const mmh3_dims* dims, const mmh3_block_weights* w, float* x, int n,
                               const mmh3_segment* segs, int n_seg, const float* pos_dev, double sigma_v,
                               double sigma_a, int modulated, const float* mods_or_null, void* workspace,
                               size_t ws_bytes, void* stream, bool profile);

// 2-D row-major tensor map, 128-byte swizzle, box {128 bytes, box_rows}.
bool make_tmap_2d(CUtensorMap* m, const void* base, int esize, uint64_t cols, uint64_t rows,
                  uint32_t box_rows);

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
inline int esize_of(int dtype) { return dtype == MMH3_BF16 ? 2 : 4; }

}  // namespace mmh3
