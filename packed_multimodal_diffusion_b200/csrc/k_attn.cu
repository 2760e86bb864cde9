// Host launcher of the tcgen05 attention kernel ("cortiq_engine/mmh3.rs",
// attention: full bidirectional softmax attention per head over the packed
// sequence; "ffai-argus 0.7.0 src/siglip.rs": attention inside each image).
#include <cmath>

#include "attn2_tc.cuh"
#include "mmh3_internal.h"

namespace mmh3 {

// Exact-fp32 attention on CUDA cores for the fp32-storage path: one thread
// per query row, 64-key tiles of K and V staged in shared memory, running
// maximum and sum (online softmax), final division by the sum.
template <int HD>
__global__ void __launch_bounds__(64) attn_f32_simt_kernel(const float* __restrict__ qkv, float* __restrict__ out,
                                                           int seq, int inner, float scale) {
  __shared__ float ks[64][HD];
  __shared__ float vs[64][HD];
  const int head = blockIdx.y;
  const int row0 = blockIdx.z * seq;
  const int qi = blockIdx.x * 64 + threadIdx.x;
  const int ld = 3 * inner;
  const bool q_ok = qi < seq;
  float q[HD], o[HD];
#pragma unroll
  for (int d = 0; d < HD; ++d) {
    q[d] = q_ok ? qkv[(size_t)(row0 + qi) * ld + head * HD + d] * scale : 0.f;
    o[d] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int k0 = 0; k0 < seq; k0 += 64) {
    __syncthreads();
    for (int e = threadIdx.x; e < 64 * HD; e += 64) {
      const int r = e / HD, d = e % HD;
      const bool ok = k0 + r < seq;
      const size_t base = (size_t)(row0 + k0 + r) * ld + head * HD + d;
      ks[r][d] = ok ? qkv[base + inner] : 0.f;
      vs[r][d] = ok ? qkv[base + 2 * inner] : 0.f;
    }
    __syncthreads();
    const int nk = seq - k0 < 64 ? seq - k0 : 64;
    for (int j = 0; j < nk; ++j) {
      float sv = 0.f;
#pragma unroll
      for (int d = 0; d < HD; ++d) sv = fmaf(q[d], ks[j][d], sv);
      const float m_new = fmaxf(m, sv);
      const float alpha = expf(m - m_new);
      const float p = expf(sv - m_new);
      l = l * alpha + p;
#pragma unroll
      for (int d = 0; d < HD; ++d) o[d] = fmaf(o[d], alpha, p * vs[j][d]);
      m = m_new;
    }
  }
  if (q_ok) {
    const float inv = l > 0.f ? 1.0f / l : 0.f;
    float* dst = out + (size_t)(row0 + qi) * inner + head * HD;
#pragma unroll
    for (int d = 0; d < HD; ++d) dst[d] = o[d] * inv;
  }
}

template <int HD>
static mmh3_status run_attn_f32(const void* qkv, int n_seq, int seq, int heads, float scale, void* out,
                                cudaStream_t s) {
  dim3 grid((seq + 63) / 64, heads, n_seq);
  attn_f32_simt_kernel<HD><<<grid, 64, 0, s>>>(static_cast<const float*>(qkv), static_cast<float*>(out), seq,
                                                heads * HD, scale); count_launch();
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MMH3_OK : cuda_fail(e, "fp32 attention launch");
}

// kv == nullptr: keys and values come from the qkv panel itself (columns
// inner and 2*inner).  Otherwise from kv [n_seq*seq_kv, 2*inner] (k at
// column 0, v at inner); the map covers exactly n_seq*seq_kv rows, so rows
// a caller padded beyond them are never read.
//
// Work units (256 query rows of one head) fill the SMs in waves, one CTA per
// SM.  When splitting the units of the last, partial wave along the keys
// shortens it (and `scratch` has room for the partial results), each tail
// unit runs as f CTAs over contiguous key ranges and attn_merge_kernel
// combines their results.
template <int HD>
static mmh3_status run_attn2(const void* qkv, int n_seq, int seq, const void* kv, int seq_kv, int heads,
                             float scale, void* out, void* scratch, size_t scratch_bytes, cudaStream_t s) {
  using Sh = Attn2Shape<HD>;
  static_assert(Sh::kSmem <= 232448, "attention shared memory above the per-CTA limit");
  const int inner = heads * HD;
  CUtensorMap tm, tkv;
  if (!make_tmap_2d(&tm, qkv, 2, (uint64_t)(3 * inner), (uint64_t)n_seq * seq, 128))
    return fail(MMH3_ERR_CUDA, "attention: cuTensorMapEncodeTiled failed");
  int k_off = inner, v_off = 2 * inner;
  if (kv != nullptr) {
    if (!make_tmap_2d(&tkv, kv, 2, (uint64_t)(2 * inner), (uint64_t)n_seq * seq_kv, 128))
      return fail(MMH3_ERR_CUDA, "attention: cuTensorMapEncodeTiled failed for K|V");
    k_off = 0;
    v_off = inner;
  } else {
    tkv = tm;
    seq_kv = seq;
  }
  auto kern = attn2_tc_kernel<HD>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Sh::kSmem);
  if (e != cudaSuccess) return cuda_fail(e, "attention smem attribute");
  const float sl2 = scale * 1.4426950408889634f;
  const int nq = (seq + 255) / 256;
  const int units = n_seq * heads * nq;
  const int sms = num_sms();
  const int tail = units % sms;
  const int kv_tiles = (seq_kv + 127) / 128;
  // f pieces per tail unit: the tail then takes ceil(tail * f / sms) rounds
  // of 1/f of a unit's time.  Take the f (at most 8, partials fitting in
  // scratch) with the fewest rounds x 1/f, the smaller f on ties, but only
  // when each piece keeps at least 32 key tiles and the tail's time drops
  // to at most 0.6 of a unit: a CTA's fixed cost (Q load, pipeline fill,
  // the partial write and the merge) eats the gain of shorter pieces.
  // Measured at 13248 keys, f = 2: -3%; at 8448 keys f = 4 (16 tiles a
  // piece): +6%; at 26496 keys f = 5 (0.8 of a unit): +1%; 32 x 1024 keys
  // f = 2 (4 tiles a piece): +7%.
  int f = 1;
  if (tail > 0 && scratch != nullptr && (reinterpret_cast<uintptr_t>(scratch) & 15) == 0) {
    double best = 1.0;
    for (int c = 2; c <= 8 && kv_tiles / c >= 32; ++c) {
      if ((size_t)tail * c * Sh::kPartBytesPerCta > scratch_bytes) break;
      const double rounds = (double)((tail * c + sms - 1) / sms) / c;
      if (rounds < best - 1e-9) {
        best = rounds;
        f = c;
      }
    }
    if (best > 0.6) f = 1;
  }
  const bool split = f >= 2;
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out);
  const int whole = split ? units - tail : units;
  if (whole > 0) {
    kern<<<whole, Sh::kThreads, Sh::kSmem, s>>>(tm, tkv, o, inner, seq, seq_kv, k_off, v_off, sl2, heads, 0, 1,
                                               nullptr, device_status_ptr(), wait_limit_ns()); count_launch();
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  }
  if (split) {
    float* part = static_cast<float*>(scratch);
    kern<<<tail * f, Sh::kThreads, Sh::kSmem, s>>>(tm, tkv, o, inner, seq, seq_kv, k_off, v_off, sl2, heads,
                                                   units - tail, f, part, device_status_ptr(), wait_limit_ns()); count_launch();
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "attention (split tail) launch");
    attn_merge_kernel<HD><<<tail * 32, 256, 0, s>>>(part, f, o, inner, seq, heads, units - tail); count_launch();
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "attention merge launch");
  }
  return MMH3_OK;
}

mmh3_status attention(int dtype, const void* qkv, int n_seq, int seq, int heads, int head_dim,
                      float scale, void* out, cudaStream_t s, void* scratch, size_t scratch_bytes) {
  if (n_seq <= 0 || seq <= 0) return MMH3_OK;
  if ((reinterpret_cast<uintptr_t>(qkv) | reinterpret_cast<uintptr_t>(out)) & 15)
    return fail(MMH3_ERR_ALIGN, "attention: pointer not 16-byte aligned");
  if (dtype == MMH3_BF16 && head_dim == 128)
    return run_attn2<128>(qkv, n_seq, seq, nullptr, 0, heads, scale, out, scratch, scratch_bytes, s);
  if (dtype == MMH3_BF16 && head_dim == 64)
    return run_attn2<64>(qkv, n_seq, seq, nullptr, 0, heads, scale, out, scratch, scratch_bytes, s);
  if (dtype == MMH3_F32 && head_dim == 64) return run_attn_f32<64>(qkv, n_seq, seq, heads, scale, out, s);
  return fail(MMH3_ERR_SHAPE, "attention: dtype %d head_dim %d unsupported", dtype, head_dim);
}

mmh3_status attention_kv(int dtype, const void* q_panel, int n_q, const void* kv, int n_kv, int heads,
                         int head_dim, float scale, void* out, cudaStream_t s, void* scratch, size_t scratch_bytes) {
  if (n_q <= 0) return MMH3_OK;
  if (n_kv <= 0) return fail(MMH3_ERR_SHAPE, "attention: %d keys", n_kv);
  if ((reinterpret_cast<uintptr_t>(q_panel) | reinterpret_cast<uintptr_t>(kv) | reinterpret_cast<uintptr_t>(out)) & 15)
    return fail(MMH3_ERR_ALIGN, "attention: pointer not 16-byte aligned");
  if (dtype == MMH3_BF16 && head_dim == 128)
    return run_attn2<128>(q_panel, 1, n_q, kv, n_kv, heads, scale, out, scratch, scratch_bytes, s);
  if (dtype == MMH3_BF16 && head_dim == 64)
    return run_attn2<64>(q_panel, 1, n_q, kv, n_kv, heads, scale, out, scratch, scratch_bytes, s);
  return fail(MMH3_ERR_UNSUPPORTED, "attention over gathered K|V: bf16 only (dtype %d, head_dim %d)", dtype,
              head_dim);
}

}  // namespace mmh3

using namespace mmh3;

extern "C" mmh3_status mmh3_attention(const void* qkv, int n_seq, int seq, int heads, int head_dim,
                                      int act_dtype, float scale, void* out, void* stream) {
  clear_error();
  if (qkv == nullptr || out == nullptr) return fail(MMH3_ERR_ARG, "attention: null pointer");
  if (heads < 1 || n_seq < 0 || seq < 0) return fail(MMH3_ERR_SHAPE, "attention: bad sizes");
  if (act_dtype != MMH3_BF16 && act_dtype != MMH3_F32) return fail(MMH3_ERR_ARG, "attention: bad dtype");
  return attention(act_dtype, qkv, n_seq, seq, heads, head_dim, scale, out, static_cast<cudaStream_t>(stream));
}

extern "C" mmh3_status mmh3_attention_ws(const void* qkv, int n_seq, int seq, int heads, int head_dim,
                                         int act_dtype, float scale, void* out, void* scratch,
                                         size_t scratch_bytes, void* stream) {
  clear_error();
  return attention(act_dtype, qkv, n_seq, seq, heads, head_dim, scale, out, static_cast<cudaStream_t>(stream),
                   scratch, scratch_bytes);
}
