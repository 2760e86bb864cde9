// Host launcher of the tcgen05 attention kernel ("cortiq_engine/mmh3.rs",
// attention: full bidirectional softmax attention per head over the packed
// sequence; "ffai-argus 0.7.0 src/siglip.rs": attention inside each image).
#include <algorithm>
#include <cmath>

#include "attn2_tc.cuh"
#include "mmh3_internal.h"

namespace mmh3 {

// Attention for the fp32-storage path on the tensor cores (tcgen05
// kind::tf32): one CTA of 128 threads per (128 query rows, head, sequence),
// key tiles of 128 processed one after another.  Per key tile:
//   1. the threads stage K [128 keys][HD] and V transposed, Vt [HD][128
//      keys], in shared memory (Q once, before the first tile);
//   2. warp 0 issues S = Q K^T into tensor memory (M 128, N 128, K HD);
//   3. thread r loads row r of S, scales it and runs the online softmax
//      (running maximum m, sum l, expf), rescales its row of O in tensor
//      memory when m grows, and writes P (fp32) to shared memory;
//   4. warp 0 issues O += P Vt^T (M 128, N HD, K 128 keys).
// Every operand is K-major: rows of 128 bytes (32 fp32) in 8-row atoms with
// the 128-byte swizzle, the 16-byte chunk c of row r at ((c ^ (r % 8)) * 16),
// written by the threads themselves (the same layout the TMA writes for the
// bf16 kernel); a K step of 8 fp32 advances the descriptor by 32 bytes.
// Keys beyond the sequence are zero-filled and masked to -inf.  After the
// last tile O / l is stored.  Waits are bounded: a CTA that gives up records
// the status word, waits (bounded) for the MMAs it issued and frees its
// tensor memory.
template <int HD>
struct AttnTf32Shape {
  static constexpr int kAtomsK = HD / 32;               // 128-byte atoms across a head
  static constexpr int kQBytes = kAtomsK * 128 * 128;   // Q or K tile
  static constexpr int kVtBytes = 4 * HD * 128;         // Vt: 4 atoms of 32 keys, HD rows
  static constexpr int kPBytes = 4 * 128 * 128;         // P: 4 atoms of 32 keys, 128 rows
  static constexpr int kQOff = 0, kKOff = kQBytes, kVtOff = 2 * kQBytes, kPOff = kVtOff + kVtBytes;
  static constexpr int kBarOff = kPOff + kPBytes;
  static constexpr int kSmem = kBarOff + 64 + 1024;     // + barriers, slot, alignment
};

__device__ __forceinline__ uint32_t sw128(uint32_t atom_base, int row, int chunk) {
  return atom_base + (uint32_t)row * 128u + ((uint32_t)(chunk ^ (row & 7)) << 4);
}

__device__ __forceinline__ void st_shared_f32(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int HD>
__global__ void __launch_bounds__(128, 1)
    attn_tf32_tc_kernel(const float* __restrict__ qkv, float* __restrict__ out, int seq, int inner, float scale,
                        DevStatus* status, uint64_t limit_ns) {
  using Sh = AttnTf32Shape<HD>;
  static_assert(HD % 32 == 0 && HD <= 128, "head_dim a multiple of 32, at most 128");
  constexpr uint32_t kIdescS = make_idesc(true, 128, 128, false, false);
  constexpr uint32_t kIdescO = make_idesc(true, 128, HD, false, false);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Sh::kBarOff);
  const uint32_t bar_s = smem_u32(bars), bar_o = smem_u32(bars + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  const int t = threadIdx.x, warp = t >> 5;
  const int head = blockIdx.y;
  const int row0 = blockIdx.z * seq;
  const int q0 = blockIdx.x * 128;
  const int ld = 3 * inner;

  if (t == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), 256);
  // Q tile: thread t writes query row q0 + t (zeros beyond the sequence)
  {
    const bool ok = q0 + t < seq;
    const float4* src = reinterpret_cast<const float4*>(qkv + (size_t)(row0 + q0 + t) * ld + head * HD);
#pragma unroll
    for (int c16 = 0; c16 < HD / 4; ++c16) {
      const float4 v = ok ? __ldg(src + c16) : make_float4(0.f, 0.f, 0.f, 0.f);
      st_shared_v4(sw128(sb + Sh::kQOff + (c16 / 8) * 16384u, t, c16 % 8),
                   make_uint4(__float_as_uint(v.x), __float_as_uint(v.y), __float_as_uint(v.z), __float_as_uint(v.w)));
    }
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_s = tmem, t_o = tmem + 128;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  float m = -INFINITY, l = 0.f;
  bool ok = true;
  int issued = 0;  // commits issued (S and O), for the drain
  const int tiles = (seq + 127) / 128;
  for (int j = 0; j < tiles && ok; ++j) {
    const int k0 = j * 128;
    {  // stage K (row = key) and Vt (row = head dim, column = key)
      const bool kok = k0 + t < seq;
      const float* base = qkv + (size_t)(row0 + k0 + t) * ld + head * HD;
      const float4* ksrc = reinterpret_cast<const float4*>(base + inner);
      const float4* vsrc = reinterpret_cast<const float4*>(base + 2 * inner);
#pragma unroll 4
      for (int c16 = 0; c16 < HD / 4; ++c16) {
        const float4 kv = kok ? __ldg(ksrc + c16) : make_float4(0.f, 0.f, 0.f, 0.f);
        st_shared_v4(sw128(sb + Sh::kKOff + (c16 / 8) * 16384u, t, c16 % 8),
                     make_uint4(__float_as_uint(kv.x), __float_as_uint(kv.y), __float_as_uint(kv.z),
                                __float_as_uint(kv.w)));
        const float4 vv = kok ? __ldg(vsrc + c16) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float ve[4] = {vv.x, vv.y, vv.z, vv.w};
        const uint32_t vt_atom = sb + Sh::kVtOff + (uint32_t)(t / 32) * (HD * 128u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int d = c16 * 4 + e;  // Vt row
          st_shared_f32(sw128(vt_atom, d, (t % 32) / 4) + (uint32_t)(t % 4) * 4u, ve[e]);
        }
      }
    }
    fence_async_smem();
    __syncthreads();
    if (warp == 0) {
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < HD / 8; ++ks) {
        const uint32_t off = (uint32_t)(ks / 4) * 16384u + (uint32_t)(ks % 4) * 32u;
        umma_ss_elect<true>(t_s, sdesc_sw128(sb + Sh::kQOff + off, 16, 1024),
                            sdesc_sw128(sb + Sh::kKOff + off, 16, 1024), kIdescS, ks > 0 ? 1u : 0u);
      }
      umma_commit_elect(bar_s);
    }
    ++issued;
    // every thread waits; the CTA leaves together if any wait ran out
    if (!__syncthreads_and(mbar_wait(bar_s, (uint32_t)(j & 1), limit_ns))) {
      if (t == 0) record_error(status, DEV_TIMEOUT_SOFTMAX, blockIdx.x);
      ok = false;
      break;
    }
    tc_fence_after();
    // row t of S, scaled, keys beyond the sequence masked: the maximum in
    // a first pass over tensor memory, the exponentials in a second
    float mt = -INFINITY;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t u[32];
      tmem_ld32(t_s + lane_off + c * 32, u);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (k0 + c * 32 + i < seq) mt = fmaxf(mt, __uint_as_float(u[i]) * scale);
    }
    const float m_new = fmaxf(m, mt);
    const float alpha = m == -INFINITY ? 0.f : expf(m - m_new);
    float psum = 0.f;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t u[32];
      tmem_ld32(t_s + lane_off + c * 32, u);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        float p4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = q * 4 + e;
          p4[e] = k0 + c * 32 + i < seq ? expf(__uint_as_float(u[i]) * scale - m_new) : 0.f;
          psum += p4[e];
        }
        st_shared_v4(sw128(sb + Sh::kPOff + (uint32_t)c * 16384u, t, q),
                     make_uint4(__float_as_uint(p4[0]), __float_as_uint(p4[1]), __float_as_uint(p4[2]),
                                __float_as_uint(p4[3])));
      }
    }
    l = l * alpha + psum;
    m = m_new;
    // rescale O when any row of the warp needs it (tcgen05.ld / st are
    // warp-collective: the whole warp runs them; other rows scale by 1);
    // the previous product has completed
    if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
      for (int c = 0; c < HD / 16; ++c) {
        uint32_t u[16];
        tmem_ld16(t_o + lane_off + c * 16, u);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
        tmem_st16(t_o + lane_off + c * 16, u);
      }
      tmem_wait_st();
    }
    tc_fence_before();
    fence_async_smem();
    __syncthreads();
    if (warp == 0) {
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < 16; ++ks) {
        const uint32_t off = (uint32_t)(ks / 4) * 16384u + (uint32_t)(ks % 4) * 32u;
        const uint32_t voff = (uint32_t)(ks / 4) * (HD * 128u) + (uint32_t)(ks % 4) * 32u;
        umma_ss_elect<true>(t_o, sdesc_sw128(sb + Sh::kPOff + off, 16, 1024),
                            sdesc_sw128(sb + Sh::kVtOff + voff, 16, 1024), kIdescO, (j > 0 || ks > 0) ? 1u : 0u);
      }
      umma_commit_elect(bar_o);
    }
    ++issued;
    if (!__syncthreads_and(mbar_wait(bar_o, (uint32_t)(j & 1), limit_ns))) {
      if (t == 0) record_error(status, DEV_TIMEOUT_SOFTMAX, blockIdx.x);
      ok = false;
      break;
    }
    tc_fence_after();
  }
  if (ok) {
    // every thread loads its row of O (warp-collective), only rows inside
    // the sequence are stored
    const float inv = l > 0.f ? 1.0f / l : 0.f;
    const bool row_ok = q0 + t < seq;
    float* dst = out + (size_t)(row0 + q0 + t) * inner + head * HD;
#pragma unroll
    for (int c = 0; c < HD / 16; ++c) {
      uint32_t u[16];
      tmem_ld16(t_o + lane_off + c * 16, u);
      tmem_wait_ld();
      if (row_ok) {
#pragma unroll
        for (int i = 0; i < 16; i += 4)
          *reinterpret_cast<float4*>(dst + c * 16 + i) =
              make_float4(__uint_as_float(u[i]) * inv, __uint_as_float(u[i + 1]) * inv,
                          __uint_as_float(u[i + 2]) * inv, __uint_as_float(u[i + 3]) * inv);
      }
    }
  } else {
    // the product whose wait ran out may still be running: wait (bounded)
    // on both barriers' next phases before tensor memory is freed
    const int j = (issued - 1) / 2;
    mbar_wait(bar_s, (uint32_t)(j & 1), limit_ns);
    if (issued % 2 == 0) mbar_wait(bar_o, (uint32_t)(j & 1), limit_ns);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int HD>
static mmh3_status run_attn_f32(const void* qkv, int n_seq, int seq, int heads, float scale, void* out,
                                cudaStream_t s) {
  using Sh = AttnTf32Shape<HD>;
  static_assert(Sh::kSmem <= 232448, "fp32 attention shared memory above the per-CTA limit");
  if ((3 * heads * HD * 4) % 16 != 0) return fail(MMH3_ERR_ALIGN, "fp32 attention: row pitch");
  auto kern = attn_tf32_tc_kernel<HD>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Sh::kSmem);
  if (e != cudaSuccess) return cuda_fail(e, "fp32 attention smem attribute");
  dim3 grid((seq + 127) / 128, heads, n_seq);
  kern<<<grid, 128, Sh::kSmem, s>>>(static_cast<const float*>(qkv), static_cast<float*>(out), seq, heads * HD, scale,
                                    device_status_ptr(), wait_limit_ns());
  count_launch();
  e = cudaGetLastError();
  return e == cudaSuccess ? MMH3_OK : cuda_fail(e, "fp32 attention launch");
}

// kv == nullptr: keys and values come from the qkv panel itself (columns
// inner and 2*inner).  Otherwise from kv [n_seq*seq_kv, 2*inner] (k at
// column 0, v at inner); the map covers exactly n_seq*seq_kv rows, so rows
// a caller padded beyond them are never read.
//
// Work units (256 query rows of one head) fill the SMs in waves, one unit
// per SM at a time.  When splitting the units of the last, partial wave
// along the keys shortens it (and `scratch` has room for the partial
// results), each tail unit runs as f items over contiguous key ranges and
// attn_merge_kernel combines their results.  The tail's items follow the
// whole units, so the SMs that finish their whole units first (they differ
// by 5-8% in speed) take them, with no launch boundary in between.
// The launch is persistent when it has a ticket counter: one CTA per SM
// takes the items in order from the counter (`ticket`, zeroed by an earlier
// kernel of the same call, or else the first kTicketBytes of scratch, zeroed
// here by a memset).  Without either, it is one CTA per item, dispatched in
// order by the hardware.
constexpr size_t kTicketBytes = 256;

template <int HD>
static mmh3_status run_attn2(const void* qkv, int n_seq, int seq, const void* kv, int seq_kv, int heads,
                             float scale, void* out, void* scratch, size_t scratch_bytes, unsigned* ticket,
                             cudaStream_t s) {
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
  if ((reinterpret_cast<uintptr_t>(scratch) & 15) != 0) scratch = nullptr;
  bool reset_ticket = false;
  if (ticket == nullptr && scratch != nullptr && scratch_bytes >= kTicketBytes) {
    ticket = static_cast<unsigned*>(scratch);
    scratch = static_cast<uint8_t*>(scratch) + kTicketBytes;
    scratch_bytes -= kTicketBytes;
    reset_ticket = true;
  }
  int f = 1;
  if (tail > 0 && scratch != nullptr) {
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
  // one launch: the whole units first, then the tail pieces (taken in order
  // from the ticket counter, or dispatched in block order without one, so
  // the SMs that finish early take the pieces)
  const int total = whole + (split ? tail * f : 0);
  float* part = split ? static_cast<float*>(scratch) : nullptr;
  if (reset_ticket) {
    e = cudaMemsetAsync(ticket, 0, sizeof(unsigned), s);
    if (e != cudaSuccess) return cuda_fail(e, "attention: ticket reset");
  }
  e = launch_pdl(kern, dim3(ticket != nullptr ? std::min(total, sms) : total), dim3(Sh::kThreads), Sh::kSmem, s, tm,
                 tkv, o, inner, seq, seq_kv, k_off, v_off, sl2, heads, whole, f, total, ticket, part,
                 device_status_ptr(), wait_limit_ns());
  count_launch();
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  if (split) {
    e = launch_pdl(attn_merge_kernel<HD>, dim3(tail * 32), dim3(256), 0, s, part, f, o, inner, seq, heads,
                   units - tail);
    count_launch();
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "attention merge launch");
  }
  return MMH3_OK;
}

mmh3_status attention(int dtype, const void* qkv, int n_seq, int seq, int heads, int head_dim,
                      float scale, void* out, cudaStream_t s, void* scratch, size_t scratch_bytes, unsigned* ticket) {
  if (n_seq <= 0 || seq <= 0) return MMH3_OK;
  if ((reinterpret_cast<uintptr_t>(qkv) | reinterpret_cast<uintptr_t>(out)) & 15)
    return fail(MMH3_ERR_ALIGN, "attention: pointer not 16-byte aligned");
  if (dtype == MMH3_BF16 && head_dim == 128)
    return run_attn2<128>(qkv, n_seq, seq, nullptr, 0, heads, scale, out, scratch, scratch_bytes, ticket, s);
  if (dtype == MMH3_BF16 && head_dim == 64)
    return run_attn2<64>(qkv, n_seq, seq, nullptr, 0, heads, scale, out, scratch, scratch_bytes, ticket, s);
  if (dtype == MMH3_F32 && head_dim == 64) return run_attn_f32<64>(qkv, n_seq, seq, heads, scale, out, s);
  return fail(MMH3_ERR_SHAPE, "attention: dtype %d head_dim %d unsupported", dtype, head_dim);
}

mmh3_status attention_kv(int dtype, const void* q_panel, int n_q, const void* kv, int n_kv, int heads,
                         int head_dim, float scale, void* out, cudaStream_t s, void* scratch, size_t scratch_bytes,
                         unsigned* ticket) {
  if (n_q <= 0) return MMH3_OK;
  if (n_kv <= 0) return fail(MMH3_ERR_SHAPE, "attention: %d keys", n_kv);
  if ((reinterpret_cast<uintptr_t>(q_panel) | reinterpret_cast<uintptr_t>(kv) | reinterpret_cast<uintptr_t>(out)) & 15)
    return fail(MMH3_ERR_ALIGN, "attention: pointer not 16-byte aligned");
  if (dtype == MMH3_BF16 && head_dim == 128)
    return run_attn2<128>(q_panel, 1, n_q, kv, n_kv, heads, scale, out, scratch, scratch_bytes, ticket, s);
  if (dtype == MMH3_BF16 && head_dim == 64)
    return run_attn2<64>(q_panel, 1, n_q, kv, n_kv, heads, scale, out, scratch, scratch_bytes, ticket, s);
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
