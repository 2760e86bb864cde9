// Persistent, warp-specialised tcgen05 GEMMs  C[M, N] = A[M, K] * B[N, K]^T
// with the block's epilogues fused in.
//
// Roles (192 threads, one CTA per SM):
//   warp 0      TMA producer: A and B tiles into a STAGES-deep smem ring
//   warp 1      MMA issuer: tcgen05.mma into one of two TMEM accumulators
//               (the whole warp runs the loop, one elected lane issues)
//   warps 2..5  epilogue: tcgen05.ld the accumulator rows, apply the fused
//               epilogue, store; the second TMEM buffer lets the next tile's
//               MMAs run under this tile's epilogue.
// gemm_tc_kernel: one CTA per 128 x BN tile, operands bf16 (kind::f16) or
// fp32 read as tf32 (kind::tf32).  gemm2_tc_kernel (further down): CTA pairs
// on one TPC computing 256 x BN tiles with tcgen05.mma.cta_group::2, bf16.
// Epilogues either store each thread's row directly or (kStageOut > 0) stage
// 128-row x 128-byte boxes in shared memory and write them with TMA tensor
// stores or tensor reduce-adds (OutStage).  Every wait is bounded
// (mbar_wait) and a timeout leaves the loops, drains in-flight copies and
// frees TMEM.
#pragma once

#include "mmh3_device.cuh"

namespace mmh3 {

template <typename T>
struct ElemTraits;
template <>
struct ElemTraits<__nv_bfloat16> {
  static constexpr bool kTf32 = false;
  static constexpr int kBytes = 2;
};
template <>
struct ElemTraits<float> {
  static constexpr bool kTf32 = true;
  static constexpr int kBytes = 4;
};

// ---------------------------------------------------------- store helpers
// Store 32 fp32 values to 32 consecutive elements of type T (16-byte aligned).
__device__ __forceinline__ void store32(__nv_bfloat16* dst, const float (&v)[32]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 u;
    u.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    u.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    u.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    u.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    d[q] = u;
  }
}
__device__ __forceinline__ void store32(float* dst, const float (&v)[32]) {
  float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int q = 0; q < 8; ++q) d[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

__device__ __forceinline__ void ld_acc32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  tmem_ld32(taddr, r);
  tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// silu(g) = g / (1 + e^-g), with the fast reciprocal division (for
// 1 + e^-g = inf it gives 0, the limit); the result is rounded to bf16.
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// The tanh form of GELU, 0.5 x (1 + tanh(u)) with u = sqrt(2/pi) (x +
// 0.044715 x^3), evaluated through the identity 0.5 (1 + tanh(u)) =
// 1 / (1 + e^(-2u)): x / (1 + e^(-2u)), one exponential and one fast
// reciprocal division, as silu above (for x far below zero the divisor
// overflows to inf and the result is 0, the limit).
__device__ __forceinline__ float gelu_tanh_f(float x) {
  const float k2 = -1.5957691216057308f;  // -2 sqrt(2/pi)
  const float u2 = k2 * x * fmaf(0.044715f * x, x, 1.0f);
  return __fdividef(x, 1.0f + __expf(u2));
}

// The same for a pair, with the multiplications and additions as packed
// f32x2 operations: x / (1 + 2^(x (c1 + c3 x^2))) with c1 = -2 sqrt(2/pi)
// log2(e) and c3 = 0.044715 c1, one ex2 and one reciprocal (both MUFU) per
// element.  The divisor is at least 1; it overflows to inf for x far below
// zero, where the reciprocal gives 0, the limit.
__device__ __forceinline__ float2 gelu_tanh_f2(float2 x) {
  const float c1 = -2.3022082f;               // -2 sqrt(2/pi) log2(e)
  const float c3 = -0.10294324f;              // 0.044715 * c1
  const float2 x2 = __fmul2_rn(x, x);
  const float2 a = __ffma2_rn(x2, make_float2(c3, c3), make_float2(c1, c1));
  const float2 u = __fmul2_rn(x, a);
  const float2 d = __fadd2_rn(make_float2(ex2_approx(u.x), ex2_approx(u.y)), make_float2(1.0f, 1.0f));
  return __fmul2_rn(x, make_float2(rcp_approx(d.x), rcp_approx(d.y)));
}

// ------------------------------------------------------------- epilogues
constexpr int kEpiParts = 1;         // epilogue warp sets (4 warps each)

template <int BN>
__device__ __forceinline__ void part_chunks(int part, int& c0, int& c1) {
  constexpr int nc = BN / 32;
  constexpr int h = (nc + kEpiParts - 1) / kEpiParts;
  c0 = part * h;
  c1 = (part + 1) * h < nc ? (part + 1) * h : nc;
}

// Epilogue warps: kEpiParts sets of four warps; the warps of one set cover
// the four TMEM lane quarters (rows), the sets split the tile's columns
// (`part`).  Contract:
//   bool operator()(tacc, row, n0, row_ok, part, wait, smem)
// tacc is the TMEM address of this thread's accumulator row (column 0),
// `wait()` blocks until the accumulator is complete (false on timeout,
// warp-uniform); loads that do not depend on the accumulator are issued
// before it.  Every tcgen05.ld is issued by all 32 lanes, also for rows
// outside the matrix.  setup() stages small parameters in shared memory.

template <int N>
__device__ __forceinline__ void ld_acc(uint32_t taddr, float (&v)[N]) {
  if constexpr (N == 32) {
    uint32_t r[32];
    tmem_ld32(taddr, r);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  } else if constexpr (N == 16) {
    uint32_t r[16];
    tmem_ld16(taddr, r);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
  } else {
    static_assert(N == 8, "8, 16 or 32 columns");
    uint32_t r[8];
    tmem_ld8(taddr, r);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
  }
}

// N consecutive values (N multiple of 8) to dst (16-byte aligned).
template <int N>
__device__ __forceinline__ void store_n(__nv_bfloat16* dst, const float (&v)[N]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < N / 8; ++q) {
    uint4 u;
    u.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    u.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    u.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    u.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    d[q] = u;
  }
}
template <int N>
__device__ __forceinline__ void store_n(float* dst, const float (&v)[N]) {
  float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int q = 0; q < N / 4; ++q) d[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

struct NoSetup {
  static constexpr int kSmemFloats = 0;
  static constexpr int kStageOut = 0;  // bytes of output staging (TMA-store epilogues)
  __device__ __forceinline__ void setup(float*, int, int) const {}
};

// Output staging for TMA-store epilogues: two buffers of one store box
// each (128 rows x 128 bytes, 128-byte swizzle).  The epilogue threads of a
// CTA write their row's 128 bytes into a free buffer, then one thread stores
// the box with a tensor store.  Compared with each thread writing its own
// row to global memory (32 cache lines per warp instruction), the tensor
// store writes whole lines and keeps the SM's L1 / shared-memory path free
// for the operand traffic of the MMAs.
struct OutStage {
  uint32_t buf0;           // shared address of buffer 0 (1024-aligned); buffer 1 at +16 KB
  const CUtensorMap* map;  // output map: box 128 bytes x 128 rows, SWIZZLE_128B
  int tid;                 // 0..127 within the epilogue group
  int r;                   // accumulator row of this thread within the tile (TMEM lane)
  int row0;                // first matrix row of the tile
  bool rows_in;            // row0 < M (a box wholly beyond M is not stored)
  uint32_t count;          // units issued so far (the same in every thread)

  // Store this thread's 128 bytes (eight 16-byte chunks) of the unit whose
  // first column is x (in elements of the map); with kAdd the unit is added
  // into global memory by a tensor reduce-add instead of overwriting it.
  template <bool kAdd = false>
  __device__ __forceinline__ void unit(const uint4 (&ch)[8], int x) {
    const uint32_t buf = buf0 + ((count & 1u) << 14);
    if (tid == 0) bulk_wait_read<1>();  // the store that last used this buffer has read it
    named_bar_sync(1, 128);
#pragma unroll
    for (int c = 0; c < 8; ++c) st_shared_v4(buf + r * 128 + ((c ^ (r & 7)) << 4), ch[c]);
    fence_proxy_async_smem();
    named_bar_sync(1, 128);
    if (tid == 0 && rows_in) {
      if constexpr (kAdd)
        tma_reduce_add_2d(map, buf, x, row0);
      else
        tma_store_2d(map, buf, x, row0);
      bulk_commit();
    }
    ++count;
  }

  // Both buffers as one 256-byte-wide unit (two boxes side by side), for
  // epilogues whose row values come out of order (the rotation pairs
  // columns j and j + 48 of a head).  begin_pair waits until the earlier
  // stores have read the buffers; put writes the 16-byte chunk `c` (0..15)
  // of this thread's row; end_pair stores both boxes at columns x, x + 64.
  __device__ __forceinline__ void begin_pair() {
    if (tid == 0) bulk_wait_read<0>();
    named_bar_sync(1, 128);
  }
  __device__ __forceinline__ void put(int c, uint4 v) {
    const uint32_t buf = buf0 + ((uint32_t)(c >> 3) << 14);
    st_shared_v4(buf + r * 128 + (((c & 7) ^ (r & 7)) << 4), v);
  }
  __device__ __forceinline__ void end_pair(int x) {
    fence_proxy_async_smem();
    named_bar_sync(1, 128);
    if (tid == 0 && rows_in) {
      tma_store_2d(map, buf0, x, row0);
      tma_store_2d(map, buf0 + 16384, x + 64, row0);
      bulk_commit();
    }
    count = 0;  // the next unit() starts on buffer 0 again
  }
};

__device__ __forceinline__ uint4 pack8_bf16(const float* v) {
  return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                    pack_bf16x2(v[6], v[7]));
}

// qkv projection: per head of the q and k planes, RMSNorm with the q_norm /
// k_norm weight, then the partial split-half 3-axis rotation from a per-row
// (cos, sin) table; v is stored as is.  Two passes over TMEM: the sum of
// squares, then the rotation in three groups of G = HD/8 pairs (one position
// axis each) and the unrotated tail -- small register footprint.
template <typename T, int HD, int BN>
struct EpiQkvNormRope {
  T* out;            // [M, N] with N = 3 * inner
  int N;
  int inner;         // heads * HD
  const float* q_norm;
  const float* k_norm;
  const float2* cs;  // frequency-major [kPairs, cs_ld] (cos, sin), or null: no rotation
  int cs_ld;         // rows of the table (the GEMM's M)
  float eps;
  static constexpr int kPairs = 3 * (HD / 8);
  static constexpr int kG = HD / 8;
  static constexpr int kSmemFloats = 2 * HD;
  static constexpr int kStageOut = 0;

  __device__ __forceinline__ void setup(float* sm, int tid, int nthreads) const {
    for (int i = tid; i < 2 * HD; i += nthreads) sm[i] = i < HD ? q_norm[i] : k_norm[i - HD];
  }

  template <class Wait>
  __device__ __forceinline__ bool operator()(uint32_t tacc, int row, int n0, bool row_ok, int part,
                                             Wait&& wait, const float* sm) const {
    constexpr int kHeadsPerPart = BN / HD / kEpiParts;
    if (!wait()) return false;
#pragma unroll 1
    for (int hh = 0; hh < kHeadsPerPart; ++hh) {
      const int g = part * kHeadsPerPart + hh;
      const int col0 = n0 + g * HD;
      if (col0 >= N) break;  // uniform across the warp
      const uint32_t th = tacc + g * HD;
      T* dst = out + (size_t)row * N + col0;
      const int which = col0 / inner;  // 0 q, 1 k, 2 v
      if (which == 2) {
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          float v[32];
          ld_acc<32>(th + c * 32, v);
          if (row_ok) store_n<32>(dst + c * 32, v);
        }
        continue;
      }
      float ss = 0.f;
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        float v[32];
        ld_acc<32>(th + c * 32, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) ss = fmaf(v[i], v[i], ss);
      }
      const float inv = rsqrtf(ss * (1.0f / HD) + eps);
      const float* w = sm + which * HD;
      if (cs != nullptr) {
#pragma unroll 1
        for (int a = 0; a < 3; ++a) {
          const int j0 = a * kG;
          float lo[kG], hi[kG];
          ld_acc<kG>(th + j0, lo);
          ld_acc<kG>(th + j0 + kPairs, hi);
          if (row_ok) {
            const float2* c2 = cs + (size_t)j0 * cs_ld + row;
#pragma unroll
            for (int i = 0; i < kG; ++i) {
              const float2 e = __ldg(c2 + (size_t)i * cs_ld);
              const float yl = lo[i] * inv * w[j0 + i];
              const float yh = hi[i] * inv * w[j0 + kPairs + i];
              lo[i] = yl * e.x - yh * e.y;
              hi[i] = yl * e.y + yh * e.x;
            }
            store_n<kG>(dst + j0, lo);
            store_n<kG>(dst + j0 + kPairs, hi);
          }
        }
        constexpr int kTail = HD - 2 * kPairs;  // 32 of 128, 16 of 64
        float t[kTail];
        ld_acc<kTail>(th + 2 * kPairs, t);
        if (row_ok) {
#pragma unroll
          for (int i = 0; i < kTail; ++i) t[i] = t[i] * inv * w[2 * kPairs + i];
          store_n<kTail>(dst + 2 * kPairs, t);
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          float v[32];
          ld_acc<32>(th + c * 32, v);
          if (row_ok) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = v[i] * inv * w[c * 32 + i];
            store_n<32>(dst + c * 32, v);
          }
        }
      }
    }
    return true;
  }
};



// The qkv epilogue with tensor-store output (pair kernel, bf16, HD = 128):
// each head's 128 columns go out as two 64-column boxes.
template <int BN>
struct EpiQkvNormRopeTma {
  int N;
  int inner;
  const float* q_norm;
  const float* k_norm;
  const float2* cs;  // frequency-major [kPairs, cs_ld] (cos, sin)
  int cs_ld;         // rows of the table (the GEMM's M)
  float eps;
  static constexpr int HD = 128;
  static constexpr int kPairs = 3 * (HD / 8);  // 48
  static constexpr int kG = HD / 8;            // 16
  static constexpr int kSmemFloats = 2 * HD;
  static constexpr int kStageOut = 32768;

  __device__ __forceinline__ void setup(float* sm, int tid, int nthreads) const {
    for (int i = tid; i < 2 * HD; i += nthreads) sm[i] = i < HD ? q_norm[i] : k_norm[i - HD];
  }

  template <class Wait>
  __device__ __forceinline__ bool operator()(uint32_t tacc, int row, int n0, bool row_ok, int, Wait&& wait,
                                             const float* sm, OutStage& st) const {
    if (!wait()) return false;
#pragma unroll 1
    for (int g = 0; g < BN / HD; ++g) {
      const int col0 = n0 + g * HD;
      if (col0 >= N) break;  // uniform over the epilogue group
      const uint32_t th = tacc + g * HD;
      const int which = col0 / inner;  // 0 q, 1 k, 2 v
      st.begin_pair();
      if (which == 2) {
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          float v[32];
          ld_acc<32>(th + c * 32, v);
#pragma unroll
          for (int q = 0; q < 4; ++q) st.put(c * 4 + q, pack8_bf16(v + 8 * q));
        }
        st.end_pair(col0);
        continue;
      }
      float ss = 0.f;
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        float v[32];
        ld_acc<32>(th + c * 32, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) ss = fmaf(v[i], v[i], ss);
      }
      const float inv = rsqrtf(ss * (1.0f / HD) + eps);
      const float* w = sm + which * HD;
#pragma unroll 1
      for (int a = 0; a < 3; ++a) {
        const int j0 = a * kG;
        float lo[kG], hi[kG];
        ld_acc<kG>(th + j0, lo);
        ld_acc<kG>(th + j0 + kPairs, hi);
        const float2* c2 = cs + (size_t)j0 * cs_ld + (row_ok ? row : 0);
#pragma unroll
        for (int i = 0; i < kG; ++i) {
          const float2 e = cs ? __ldg(c2 + (size_t)i * cs_ld) : make_float2(1.f, 0.f);
          const float yl = lo[i] * inv * w[j0 + i];
          const float yh = hi[i] * inv * w[j0 + kPairs + i];
          lo[i] = yl * e.x - yh * e.y;
          hi[i] = yl * e.y + yh * e.x;
        }
        st.put(j0 / 8, pack8_bf16(lo));
        st.put(j0 / 8 + 1, pack8_bf16(lo + 8));
        st.put((j0 + kPairs) / 8, pack8_bf16(hi));
        st.put((j0 + kPairs) / 8 + 1, pack8_bf16(hi + 8));
      }
      float t[HD - 2 * kPairs];  // the 32 unrotated dims
      ld_acc<32>(th + 2 * kPairs, t);
#pragma unroll
      for (int i = 0; i < 32; ++i) t[i] = t[i] * inv * w[2 * kPairs + i];
#pragma unroll
      for (int q = 0; q < 4; ++q) st.put(2 * kPairs / 8 + q, pack8_bf16(t + 8 * q));
      st.end_pair(col0);
    }
    return true;
  }
};

// out = act(acc + bias), bf16, with tensor-store output (pair kernel).
// bias must be 16-byte aligned (it is read as float4).
template <int BN, int MODE>
struct EpiBiasActTma : NoSetup {
  static constexpr int kStageOut = 32768;
  int N;
  const float* bias;

  template <class Wait>
  __device__ __forceinline__ bool operator()(uint32_t tacc, int, int n0, bool, int, Wait&& wait, const float*,
                                             OutStage& st) const {
    if (!wait()) return false;
#pragma unroll 1
    for (int u = 0; u < BN / 64; ++u) {
      const int col = n0 + u * 64;
      if (col >= N) break;
      // both 32-column halves of the unit in flight before one wait
      uint32_t r[2][32];
      tmem_ld32(tacc + u * 64, r[0]);
      tmem_ld32(tacc + u * 64 + 32, r[1]);
      tmem_wait_ld();
      uint4 ch[8];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float v[32];
        const float4* b4 = reinterpret_cast<const float4*>(bias + col + h * 32);  // 16-byte aligned
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 b = __ldg(b4 + i / 4);
          float2 t0 = __fadd2_rn(make_float2(__uint_as_float(r[h][i]), __uint_as_float(r[h][i + 1])),
                                 make_float2(b.x, b.y));
          float2 t1 = __fadd2_rn(make_float2(__uint_as_float(r[h][i + 2]), __uint_as_float(r[h][i + 3])),
                                 make_float2(b.z, b.w));
          if (MODE == 1) {
            t0 = gelu_tanh_f2(t0);
            t1 = gelu_tanh_f2(t1);
          }
          v[i] = t0.x;
          v[i + 1] = t0.y;
          v[i + 2] = t1.x;
          v[i + 3] = t1.y;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) ch[h * 4 + q] = pack8_bf16(v + 8 * q);
      }
      st.unit(ch, col);
    }
    return true;
  }
};

// x[row, :] += gate[row] * acc (the gated residual; gate = chunk of the
// token's modulation row, found through the segment table), or x += acc when
// mods is null, or x += acc + bias (the encoder layer's biased residual).
// The x and gate/bias values of a chunk are loaded before the accumulator
// chunk is read, and the next chunk's before the current one is stored.
template <int BN, bool BIAS>
struct EpiResidual : NoSetup {
  float* x;          // [M, N] fp32, in place
  int N;
  const float* mods; // [rows, mods_stride] or null (gated form)
  int mods_stride;
  int chunk_off;     // chunk * hidden
  SegRows seg;
  const float* bias; // [N] (biased form)

  __device__ __forceinline__ void load_x(int row, int col, bool row_ok, float4 (&xv)[8]) const {
    if (row_ok) {
      const float4* xp = reinterpret_cast<const float4*>(x + (size_t)row * N + col);
#pragma unroll
      for (int q = 0; q < 8; ++q) xv[q] = xp[q];
    }
  }

  template <class Wait>
  __device__ __forceinline__ bool operator()(uint32_t tacc, int row, int n0, bool row_ok, int part,
                                             Wait&& wait, const float*) const {
    const float* g = nullptr;
    if (BIAS) g = bias;
    else if (mods != nullptr) g = mods + (size_t)seg_row_checked(seg, row) * mods_stride + chunk_off;
    int c0, c1;
    part_chunks<BN>(part, c0, c1);
    float4 xa[8];
    if (c0 < c1 && n0 + c0 * 32 < N) load_x(row, n0 + c0 * 32, row_ok, xa);
    if (!wait()) return false;
#pragma unroll 1
    for (int c = c0; c < c1; ++c) {
      const int col = n0 + c * 32;
      if (col >= N) break;
      float4 gv[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        gv[q] = g ? __ldg(reinterpret_cast<const float4*>(g + col) + q) : make_float4(1.f, 1.f, 1.f, 1.f);
      float v[32];
      ld_acc<32>(tacc + c * 32, v);
      float4 xb[8];
      const bool next = c + 1 < c1 && col + 32 < N;
      if (next) load_x(row, col + 32, row_ok, xb);
      if (row_ok) {
        float4* xp = reinterpret_cast<float4*>(x + (size_t)row * N + col);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float4 o = xa[q];
          if (BIAS) {
            o.x += v[4 * q + 0] + gv[q].x;
            o.y += v[4 * q + 1] + gv[q].y;
            o.z += v[4 * q + 2] + gv[q].z;
            o.w += v[4 * q + 3] + gv[q].w;
          } else {
            o.x = fmaf(gv[q].x, v[4 * q + 0], o.x);
            o.y = fmaf(gv[q].y, v[4 * q + 1], o.y);
            o.z = fmaf(gv[q].z, v[4 * q + 2], o.z);
            o.w = fmaf(gv[q].w, v[4 * q + 3], o.w);
          }
          xp[q] = o;
        }
      }
      if (next) {
#pragma unroll
        for (int q = 0; q < 8; ++q) xa[q] = xb[q];
      }
    }
    return true;
  }
};

template <int BN>
using EpiGatedResidual = EpiResidual<BN, false>;
template <int BN>
using EpiBiasResidual = EpiResidual<BN, true>;

// x += gate * acc (or x += acc + bias) without reading x: each 32-column
// unit of gate * acc is staged in shared memory and added into x by a
// tensor reduce-add, so x passes neither through shared memory nor through
// the registers, and each element of x is updated exactly once.  (Staging
// x itself, loaded, updated and stored back, moved four 16 KB passes
// through shared memory per unit against the operand traffic of the
// MMAs, which a 256-wide pair tile already brings near shared memory's
// bandwidth; measured: out 3.5% and fc2 1.8% slower.)
template <int BN, bool BIAS>
struct EpiResidualTma : NoSetup {
  static constexpr int kStageOut = 32768;
  static constexpr int kUnits = BN / 32;
  int N;
  const float* mods;
  int mods_stride;
  int chunk_off;
  SegRows seg;
  const float* bias;

  template <class Wait>
  __device__ __forceinline__ bool operator()(uint32_t tacc, int row, int n0, bool, int, Wait&& wait,
                                             const float*, OutStage& st) const {
    const int units = (N - n0) / 32 < kUnits ? (N - n0) / 32 : kUnits;
    if (!wait()) return false;
    if (!st.rows_in) return true;
    const float* g = nullptr;
    if (BIAS) g = bias;
    else if (mods != nullptr) g = mods + (size_t)seg_row_checked(seg, row) * mods_stride + chunk_off;
#pragma unroll 1
    for (int u = 0; u < units; ++u) {
      const int col = n0 + u * 32;
      float v[32];
      ld_acc<32>(tacc + u * 32, v);
      uint4 ch[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 gv = g ? __ldg(reinterpret_cast<const float4*>(g + col) + q) : make_float4(1.f, 1.f, 1.f, 1.f);
        float4 o;
        if (BIAS)
          o = make_float4(v[4 * q + 0] + gv.x, v[4 * q + 1] + gv.y, v[4 * q + 2] + gv.z, v[4 * q + 3] + gv.w);
        else
          o = make_float4(gv.x * v[4 * q + 0], gv.y * v[4 * q + 1], gv.z * v[4 * q + 2], gv.w * v[4 * q + 3]);
        ch[q] = make_uint4(__float_as_uint(o.x), __float_as_uint(o.y), __float_as_uint(o.z), __float_as_uint(o.w));
      }
      st.template unit<true>(ch, col);
    }
    return true;
  }
};

// fc1 + SwiGLU: the weight rows are interleaved so that tile columns
// [0, BN/2) are gate rows and [BN/2, BN) the matching up rows; the output
// column block is n0 / 2.
template <typename T, int BN>
struct EpiSwiGLU : NoSetup {
  T* out;  // [M, F]
  int F;

  template <class Wait>
  __device__ __forceinline__ bool operator()(uint32_t tacc, int row, int n0, bool row_ok, int part,
                                             Wait&& wait, const float*) const {
    if (!wait()) return false;
    constexpr int np = BN / 64;  // chunk pairs
    const int f0 = n0 / 2;
#pragma unroll 1
    for (int c = part * (np / kEpiParts); c < (part + 1) * (np / kEpiParts); ++c) {
      const int f = f0 + c * 32;
      if (f >= F) break;
      float gt[32], u[32];
      ld_acc<32>(tacc + c * 32, gt);
      ld_acc<32>(tacc + BN / 2 + c * 32, u);
      if (row_ok) {
#pragma unroll
        for (int i = 0; i < 32; ++i) gt[i] = silu_f(gt[i]) * u[i];
        store_n<32>(out + (size_t)row * F + f, gt);
      }
    }
    return true;
  }
};

// fc1 + SwiGLU with the output written by tensor stores (pair kernel):
// each 256-column tile gives 128 outputs, two store units of 64 bf16.
template <int BN>
struct EpiSwiGLUTma : NoSetup {
  static constexpr int kStageOut = 32768;
  int F;

  template <class Wait>
  __device__ __forceinline__ bool operator()(uint32_t tacc, int, int n0, bool, int, Wait&& wait, const float*,
                                             OutStage& st) const {
    if (!wait()) return false;
#pragma unroll 1
    for (int u = 0; u < BN / 128; ++u) {
      uint4 ch[8];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float gt[32], up[32];
        ld_acc<32>(tacc + u * 64 + h * 32, gt);
        ld_acc<32>(tacc + BN / 2 + u * 64 + h * 32, up);
#pragma unroll
        for (int i = 0; i < 32; ++i) gt[i] = silu_f(gt[i]) * up[i];
#pragma unroll
        for (int q = 0; q < 4; ++q) ch[h * 4 + q] = pack8_bf16(gt + 8 * q);
      }
      st.unit(ch, n0 / 2 + u * 64);
    }
    return true;
  }
};

// out = act(acc + bias) for the unmodulated encoder layer and the output
// heads.  MODE 0: identity, 1: tanh-GELU, 2: negate (velocity sign).
template <typename T, int BN, int MODE>
struct EpiBiasAct : NoSetup {
  T* out;
  int N;
  const float* bias;

  template <class Wait>
  __device__ __forceinline__ bool operator()(uint32_t tacc, int row, int n0, bool row_ok, int part,
                                             Wait&& wait, const float*) const {
    if (!wait()) return false;
    int c0, c1;
    part_chunks<BN>(part, c0, c1);
#pragma unroll 1
    for (int c = c0; c < c1; ++c) {
      const int col = n0 + c * 32;
      if (col >= N) break;
      float v[32];
      ld_acc<32>(tacc + c * 32, v);
      if (row_ok) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          float t = v[i] + __ldg(bias + col + i);
          if (MODE == 1) t = gelu_tanh_f(t);
          if (MODE == 2) t = -t;
          v[i] = t;
        }
        store_n<32>(out + (size_t)row * N + col, v);
      }
    }
    return true;
  }
};

// ------------------------------------------------------------------ kernel
// Tile order: groups of group_m row tiles, all column tiles of a group
// before the next group, row tiles fastest within a group.  The persistent
// CTAs work on a window of consecutive tiles, so a group's A panel is
// reused from L2 by all its column tiles while B is swept once per group;
// the host sizes the group (group_m_for).
__device__ __forceinline__ void tile_coords(int tile, int m_tiles, int n_tiles, int group_m, int& mt, int& nt) {
  const int per_group = group_m * n_tiles;
  const int g = tile / per_group;
  const int first_m = g * group_m;
  const int gm = (m_tiles - first_m) < group_m ? (m_tiles - first_m) : group_m;
  const int t = tile - g * per_group;
  mt = first_m + t % gm;
  nt = t / gm;
}

template <int BN>
struct GemmShape {
  static constexpr int BM = 128;
  static constexpr int kABytes = BM * 128;  // 128 rows of 128 bytes
  static constexpr int kBBytes = BN * 128;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128
                                   : (2 * BN <= 256) ? 256 : 512;
};

constexpr int kEpiSmemBytes = 2048;  // staged epilogue parameters
constexpr int kGemmThreads = 64 + 128 * kEpiParts;  // producer, MMA, epilogue

// stages | output staging | barriers | epilogue parameters
template <int BN, int STAGES, int OUT = 0>
constexpr int gemm_smem_bytes() {
  return STAGES * GemmShape<BN>::kStageBytes + OUT + 1024 /*align*/ + 256 /*barriers*/ + kEpiSmemBytes;
}

template <typename T, int BN, int STAGES, class Epi>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, int M, int N, int K, int group_m, Epi epi,
                   DevStatus* status, uint64_t limit_ns) {
  using Sh = GemmShape<BN>;
  constexpr bool kTf32 = ElemTraits<T>::kTf32;
  constexpr int kOut = Epi::kStageOut;
  static_assert(kOut == 0 || kOut == 32768, "output staging is two 16 KB boxes");
  constexpr int kBK = 128 / ElemTraits<T>::kBytes;  // K elements per stage
  constexpr uint32_t kIdesc = make_idesc(kTf32, 128, BN, false, false);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t stage_out = smem_u32(smem + STAGES * Sh::kStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * Sh::kStageBytes + kOut);
  // bars: full[STAGES] empty[STAGES] tfull[2] tempty[2] drain; then the
  // TMEM address slot and the CTA's abort flag
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* epi_smem = reinterpret_cast<float*>(smem + STAGES * Sh::kStageBytes + kOut + 256);
  static_assert(Epi::kSmemFloats * 4 <= kEpiSmemBytes, "epilogue parameters exceed their smem area");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 32 * (kGemmThreads / 32 - 2));
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch(&tmA);
    tma_prefetch(&tmB);
    if (kOut > 0) tma_prefetch(&tmC);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), Sh::kTmemCols);
  if (warp >= 2) epi.setup(epi_smem, threadIdx.x - 64, kGemmThreads - 64);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait();

  const int m_tiles = (M + Sh::BM - 1) / Sh::BM;
  const int n_tiles = (N + BN - 1) / BN;
  const int num_tiles = m_tiles * n_tiles;
  const int k_blocks = (K + kBK - 1) / kBK;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      const bool chk = status != nullptr && status->check != 0;
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;  // stages whose copies may still be in flight
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        int mt, nt;
        tile_coords(tile, m_tiles, n_tiles, group_m, mt, nt);
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (*abort_flag || !mbar_wait(empty_bar(stage), phase ^ 1u, limit_ns)) {
            if (!*abort_flag) record_error(status, DEV_TIMEOUT_PRODUCER, tile);
            *abort_flag = 1;
            ok = false;
            break;
          }
          if (!tma_coords_ok(status, chk, kb * kBK, mt * Sh::BM, ElemTraits<T>::kBytes) ||
              !tma_coords_ok(status, chk, kb * kBK, nt * BN, ElemTraits<T>::kBytes)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          const uint32_t sa = sbase + stage * Sh::kStageBytes;
          mbar_expect_tx(full_bar(stage), Sh::kStageBytes);
          tma_load_2d(sa, &tmA, full_bar(stage), kb * kBK, mt * Sh::BM);
          tma_load_2d(sa + Sh::kABytes, &tmB, full_bar(stage), kb * kBK, nt * BN);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // Drain: every issued stage's copy must land before the CTA exits.
        // The most recent min(issued, STAGES) stages may be outstanding.
        int s = stage;
        uint32_t ph = phase;
        const int outstanding = issued < STAGES ? issued : STAGES;
        for (int i = 0; i < outstanding; ++i) {
          if (--s < 0) {
            s = STAGES - 1;
            ph ^= 1u;
          }
          mbar_wait(full_bar(s), ph, limit_ns);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: the whole warp runs the loop and its
    // waits (warp-uniform descriptors and addresses); the lane elect.sync
    // picks, always the same, issues every MMA and commit.
    const uint64_t d_base = sdesc_sw128(sbase, 16, 1024);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      if (!__all_sync(0xffffffffu, mbar_wait_ab(tempty_bar(acc), acc_phase ^ 1u, limit_ns, abort_flag))) {
        if (lane == 0 && !*abort_flag) record_error(status, DEV_TIMEOUT_MMA, 1000 + tile);
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * BN;
      for (int kb = 0; kb < k_blocks; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait_ab(full_bar(stage), phase, limit_ns, abort_flag))) {
          if (lane == 0 && !*abort_flag) record_error(status, DEV_TIMEOUT_MMA, tile);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t ad = d_base + (uint64_t)((stage * Sh::kStageBytes) >> 4);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          umma_ss_elect<kTf32>(d_tmem, ad + 2 * ks, ad + (Sh::kABytes >> 4) + 2 * ks, kIdesc,
                               (kb | ks) != 0 ? 1u : 0u);
        umma_commit_elect(empty_bar(stage));
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      umma_commit_elect(tfull_bar(acc));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    // Drain: wait until every MMA this warp issued has completed before
    // TMEM is released (a commit tracks all prior MMAs of the thread).
    if (!ok) {
      __syncwarp();
      *abort_flag = 1;
      umma_commit_elect(drain_bar);
      mbar_wait(drain_bar, 0, limit_ns);
    }
  } else {
    // ---------------- epilogue warps 2..5: lane quarter warp % 4
    const int lgrp = warp & 3;
    const int part = (warp - 2) >> 2;
    const uint32_t lane_off = (uint32_t)(lgrp * 32) << 16;
    OutStage ost{stage_out, &tmC, (int)threadIdx.x - 64, lgrp * 32 + lane, 0, false, 0u};
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      int mt, nt;
      tile_coords(tile, m_tiles, n_tiles, group_m, mt, nt);
      const int row = mt * Sh::BM + lgrp * 32 + lane;
      // warp-uniform (the TMEM loads are warp-collective); group-uniform for
      // staged output (its named barriers need all 128 threads)
      auto wait = [&]() -> bool {
        bool fail = *abort_flag || !mbar_wait(tfull_bar(acc), acc_phase, limit_ns);
        if constexpr (kOut > 0) fail = named_bar_or(2, 128, fail);
        if (__any_sync(0xffffffffu, fail)) {
          if (lane == 0 && !*abort_flag) record_error(status, DEV_TIMEOUT_EPILOGUE, tile);
          *abort_flag = 1;
          return false;
        }
        tc_fence_after();
        return true;
      };
      bool go;
      if constexpr (kOut > 0) {
        ost.row0 = mt * Sh::BM;
        ost.rows_in = ost.row0 < M;
        go = epi(tmem_base + acc * BN + lane_off, row, nt * BN, row < M, part, wait, epi_smem, ost);
      } else {
        go = epi(tmem_base + acc * BN + lane_off, row, nt * BN, row < M, part, wait, epi_smem);
      }
      if (!go) break;
      tc_fence_before();
      mbar_arrive(tempty_bar(acc));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if constexpr (kOut > 0) {
      if (ost.tid == 0) bulk_wait_all();  // the tensor stores and adds have written global memory
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Sh::kTmemCols);
  }
}


// ======================================================= CTA-pair variant
// The same GEMM on clusters of two CTAs (one TPC): a pair computes a
// 256 x BN tile with tcgen05.mma.cta_group::2 (M = 256).  Each CTA loads its
// own 128 rows of A and half of B's BN rows (BN/2) per stage, so a CTA's
// shared-memory operand traffic per MMA is A + B/2 instead of A + B.
//   both CTAs   warp 0: TMA of their own A rows / B half; completion is
//               counted on the LEADER's full barrier (the leader expects the
//               bytes of both); each CTA waits on its own empty barrier.
//   leader      warp 1: the MMAs, descriptors on its own shared-memory
//               offsets (the hardware reads the same offsets in the peer);
//               commits multicast to both CTAs' empty / accumulator-full
//               barriers.
//   both CTAs   warps 2..5: epilogue of their own 128 accumulator rows; the
//               release arrives on the leader's accumulator-empty barrier
//               (256 arrivals).
// The tensor memory is allocated and freed by warp 1 of both CTAs
// together.  Loads carry no multicast.  Every wait is bounded.
template <int BN>
struct Gemm2Shape {
  static constexpr int BM = 128;                 // rows per CTA, 256 per pair
  static constexpr int kABytes = BM * 128;
  static constexpr int kBRows = BN / 2;          // B rows held by each CTA
  static constexpr int kBBytes = kBRows * 128;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = (2 * BN <= 256) ? 256 : 512;
  static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "pair tile width");
};

// stages | output staging | barriers | epilogue parameters
template <int BN, int STAGES, class Epi>
constexpr int gemm2_smem_bytes() {
  return STAGES * Gemm2Shape<BN>::kStageBytes + Epi::kStageOut + 1024 /*align*/ + 256 /*barriers*/ +
         ((Epi::kSmemFloats * 4 + 255) / 256) * 256;
}

template <int BN, int STAGES, class Epi>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm2_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmC, int M, int N, int K, int group_m, Epi epi,
                    DevStatus* status,
                    uint64_t limit_ns) {
  using Sh = Gemm2Shape<BN>;
  constexpr int kBK = 64;  // bf16 K elements per stage (128 bytes)
  constexpr uint32_t kIdesc = make_idesc(false, 256, BN, false, false);
  constexpr int kOut = Epi::kStageOut;
  static_assert(kOut == 0 || kOut == 32768, "output staging is two 16 KB boxes");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t stage_out = smem_u32(smem + STAGES * Sh::kStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * Sh::kStageBytes + kOut);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* epi_smem = reinterpret_cast<float*>(smem + STAGES * Sh::kStageBytes + kOut + 256);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int st) { return bar0 + 8u * st; };
  auto empty_bar = [&](int st) { return bar0 + 8u * (STAGES + st); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  constexpr int kEpiThreads = kGemmThreads - 64;

  if (threadIdx.x == 0) {
    for (int st = 0; st < STAGES; ++st) {
      mbar_init(full_bar(st), 1);
      mbar_init(empty_bar(st), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 2 * kEpiThreads);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch(&tmA);
    tma_prefetch(&tmB);
    if (kOut > 0) tma_prefetch(&tmC);
  }
  if (warp == 1) tmem_alloc_pair(smem_u32(tmem_slot), Sh::kTmemCols);
  if (warp >= 2) epi.setup(epi_smem, threadIdx.x - 64, kEpiThreads);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive or TMA
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait();

  const int m_tiles = (M + 2 * Sh::BM - 1) / (2 * Sh::BM);
  const int n_tiles = (N + BN - 1) / BN;
  const int num_tiles = m_tiles * n_tiles;
  const int k_blocks = (K + kBK - 1) / kBK;
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs)
      const bool chk = status != nullptr && status->check != 0;
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += n_pairs) {
        int mt, nt;
        tile_coords(tile, m_tiles, n_tiles, group_m, mt, nt);
        const int a_row = mt * 2 * Sh::BM + (int)rank * Sh::BM;
        const int b_row = nt * BN + (int)rank * Sh::kBRows;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (*abort_flag || !mbar_wait(empty_bar(stage), phase ^ 1u, limit_ns)) {
            if (!*abort_flag) record_error(status, DEV_TIMEOUT_PRODUCER, tile);
            *abort_flag = 1;
            ok = false;
            break;
          }
          if (!tma_coords_ok(status, chk, kb * kBK, a_row, 2) || !tma_coords_ok(status, chk, kb * kBK, b_row, 2)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          const uint32_t sa = sbase + stage * Sh::kStageBytes;
          const uint32_t fb = mapa_shared(full_bar(stage), 0);
          if (leader) mbar_expect_tx(full_bar(stage), 2 * Sh::kStageBytes);
          tma_load_2d_pair(sa, &tmA, fb, kb * kBK, a_row);
          tma_load_2d_pair(sa + Sh::kABytes, &tmB, fb, kb * kBK, b_row);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && leader) {
        // The leader's full barriers count both CTAs' copies: wait (bounded)
        // for the outstanding stages before the pair leaves.
        int st = stage;
        uint32_t ph = phase;
        const int outstanding = issued < STAGES ? issued : STAGES;
        for (int i = 0; i < outstanding; ++i) {
          if (--st < 0) {
            st = STAGES - 1;
            ph ^= 1u;
          }
          mbar_wait(full_bar(st), ph, limit_ns);
        }
      }
    }
  } else if (warp == 1) {
    if (leader) {
      // ---------------- MMA issuer (leader only): the whole warp runs the
      // loop and its waits; the lane elect.sync picks issues (as in the
      // single-CTA kernel).
      const uint64_t d_base = sdesc_sw128(sbase, 16, 1024);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += n_pairs) {
        const bool got = !*abort_flag && mbar_wait_cluster(tempty_bar(acc), acc_phase ^ 1u, limit_ns);
        if (!__all_sync(0xffffffffu, got)) {
          if (lane == 0 && !*abort_flag) record_error(status, DEV_TIMEOUT_MMA, 1000 + tile);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!__all_sync(0xffffffffu, mbar_wait_ab(full_bar(stage), phase, limit_ns, abort_flag))) {
            if (lane == 0 && !*abort_flag) record_error(status, DEV_TIMEOUT_MMA, tile);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = d_base + (uint64_t)((stage * Sh::kStageBytes) >> 4);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            umma_ss_pair_elect(d_tmem, ad + 2 * ks, ad + (Sh::kABytes >> 4) + 2 * ks, kIdesc,
                               (kb | ks) != 0 ? 1u : 0u);
          umma_commit_pair_elect(empty_bar(stage));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair_elect(tfull_bar(acc));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok) {
        __syncwarp();
        *abort_flag = 1;
        if (lane == 0) umma_commit_pair_local(drain_bar);
        mbar_wait(drain_bar, 0, limit_ns);
      }
    }
  } else {
    // ---------------- epilogue warps 2..5: this CTA's 128 rows
    const int lgrp = warp & 3;
    const int part = (warp - 2) >> 2;
    const uint32_t lane_off = (uint32_t)(lgrp * 32) << 16;
    OutStage ost{stage_out, &tmC, (int)threadIdx.x - 64, lgrp * 32 + lane, 0, false, 0u};
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < num_tiles; tile += n_pairs) {
      int mt, nt;
      tile_coords(tile, m_tiles, n_tiles, group_m, mt, nt);
      const int row0 = mt * 2 * Sh::BM + (int)rank * Sh::BM;
      const int row = row0 + lgrp * 32 + lane;
      // The decision to go on is uniform over the warp (TMEM loads are
      // warp-collective) and, for staged output, over the whole epilogue
      // group (its named barriers need all 128 threads).
      auto wait = [&]() -> bool {
        bool fail = *abort_flag || !mbar_wait_cluster(tfull_bar(acc), acc_phase, limit_ns);
        if constexpr (kOut > 0) fail = named_bar_or(2, 128, fail);
        if (__any_sync(0xffffffffu, fail)) {
          if (lane == 0 && !*abort_flag) record_error(status, DEV_TIMEOUT_EPILOGUE, tile);
          *abort_flag = 1;
          return false;
        }
        tc_fence_after();
        return true;
      };
      bool go;
      if constexpr (kOut > 0) {
        ost.row0 = row0;
        ost.rows_in = row0 < M;
        go = epi(tmem_base + acc * BN + lane_off, row, nt * BN, row < M, part, wait, epi_smem, ost);
      } else {
        go = epi(tmem_base + acc * BN + lane_off, row, nt * BN, row < M, part, wait, epi_smem);
      }
      if (!go) break;
      tc_fence_before();
      mbar_arrive_cluster(mapa_shared(tempty_bar(acc), 0));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if constexpr (kOut > 0) {
      if (ost.tid == 0) bulk_wait_all();  // the tensor stores and adds have written global memory
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no remote arrive, copy or MMA of either CTA is pending
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, Sh::kTmemCols);
  }
}

}  // namespace mmh3
