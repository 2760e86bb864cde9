// Memory-bound kernels of the block: the prologue (adaLN curve evaluation
// and the rotary (cos, sin) table in one launch), the fused
// segment-gather RMSNorm + modulate, the
// encoder layer's LayerNorm and the weight-preparation copies; plus the
// device status word written by bounded waits.
//
// Sources: "cortiq_engine/mmh3.rs" (cortiq-engine 0.5.72) -- Adaln::eval,
// rms_norm_into, norm_rows, modulate, rope_angles; "inferencelayer 0.2.1
// src/encoder_cpu.rs" -- layer_norm_rows (two-pass variance).
#include <cmath>
#include <cstdio>

#include "mmh3_device.cuh"
#include "mmh3_internal.h"

namespace mmh3 {

// ------------------------------------------------------------ status word
__device__ DevStatus g_dev_status;

// The status word of the current device; the first lookup on a device also
// writes the check-mode flag into it (MMH3_CHECK=1 or mmh3_set_check).
DevStatus* device_status_ptr() {
  static DevStatus* ptrs[64] = {nullptr};
  static int flag_written[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (ptrs[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dev_status) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<DevStatus*>(p);
    flag_written[dev] = -1;
  }
  const int want = check_mode() ? 1 : 0;
  if (flag_written[dev] != want) {
    if (cudaMemcpy(&ptrs[dev]->check, &want, sizeof(int), cudaMemcpyHostToDevice) == cudaSuccess)
      flag_written[dev] = want;
  }
  return ptrs[dev];
}

// ------------------------------------------------ workspace canaries
// MMH3_CHECK mode: a 256-byte canary follows each workspace region; fill
// writes a position-dependent pattern, verify records DEV_CHECK_CANARY
// (site: kernel * 16 + region) for the first word found changed.
__global__ void canary_kernel(CanaryList l, int verify, int kernel_id, DevStatus* st) {
  for (int i = threadIdx.x; i < l.n * (kCanaryBytes / 4); i += blockDim.x) {
    uint32_t* p = l.p[i / (kCanaryBytes / 4)] + (i % (kCanaryBytes / 4));
    const uint32_t want = 0xC0FFEE5Au ^ (uint32_t)i;
    if (!verify)
      *p = want;
    else if (*p != want)
      record_error(st, DEV_CHECK_CANARY, kernel_id * 16 + i / (kCanaryBytes / 4));
  }
}

cudaError_t launch_canary(const CanaryList& l, bool verify, int kernel_id, cudaStream_t s) {
  if (l.n == 0) return cudaSuccess;
  canary_kernel<<<1, 256, 0, s>>>(l, verify ? 1 : 0, kernel_id, device_status_ptr());
  count_launch();
  return cudaGetLastError();
}

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (cached[dev] == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = v > 0 ? v : 148;
  }
  return cached[dev];
}

// -------------------------------------------------------------- K1 adaLN
// out[s*rows_per_slot + r] = w[row] . c_s + b[row], c_s the interpolated
// curve coordinates of timestep slot s (rank <= 32).
struct CurveArgs {
  int i0[2];
  float f[2];
};

__global__ void __launch_bounds__(256) adaln_kernel(const float* __restrict__ w,
                                                    const float* __restrict__ b,
                                                    const float* __restrict__ table, int rank,
                                                    int rows_per_slot, int n_ts, CurveArgs ca,
                                                    float* __restrict__ out) {
  __shared__ float c[2][32];
  if (threadIdx.x < n_ts * rank) {
    const int s = threadIdx.x / rank, k = threadIdx.x % rank;
    const float a = table[ca.i0[s] * rank + k];
    const float bb = table[(ca.i0[s] + 1) * rank + k];
    const float f = ca.f[s];
    c[s][k] = (1.0f - f) * a + f * bb;
  }
  __syncthreads();
  const int total = n_ts * rows_per_slot;
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < total; r += gridDim.x * blockDim.x) {
    const int s = r / rows_per_slot;
    const float* wr = w + (size_t)r * rank;
    float acc = 0.f;
    if (rank == 24) {
      const float4* w4 = reinterpret_cast<const float4*>(wr);
#pragma unroll
      for (int q = 0; q < 6; ++q) {
        const float4 v = __ldg(w4 + q);
        acc = fmaf(v.x, c[s][4 * q + 0], acc);
        acc = fmaf(v.y, c[s][4 * q + 1], acc);
        acc = fmaf(v.z, c[s][4 * q + 2], acc);
        acc = fmaf(v.w, c[s][4 * q + 3], acc);
      }
    } else {
      for (int k = 0; k < rank; ++k) acc = fmaf(__ldg(wr + k), c[s][k], acc);
    }
    out[r] = acc + __ldg(b + r);
  }
}

// ------------------------------------------------ the block's prologue
// One launch computes what a block (or a whole stack) reads before its
// first RMSNorm: the adaLN modulation rows of up to kAdalnBatch blocks and
// the rotation (cos, sin) table.  Work items are one warp each: the first
// n_ab * (n_ts * rows_per_slot / 32) items evaluate 32 consecutive
// modulation rows of one block; the rest fill 256 table entries.
//  - adaLN ("cortiq_engine/mmh3.rs", Adaln::eval): the warp's 32 basis rows
//    are one contiguous run of 32 * rank floats, read as float4 at
//    lane + 32 q (coalesced); each float4 is dotted with its four curve
//    coordinates, and a row's rank / 4 partial dots are added from shared
//    memory, then the bias; the 32 results are one coalesced store.
//  - rotation table ("cortiq_engine/mmh3.rs", rope_angles): cs[i, j] =
//    (cos a, sin a), a = pos[i, j / K] * inv_freq[j % K], the product taken
//    in fp64 and rounded to fp32, then CUDA's sincosf.
struct InvFreq {
  float v[32];
};

template <int K>  // rotation frequencies per axis (8 or 16); 0: no table
__global__ void __launch_bounds__(256, 4)
    prologue_kernel(AdalnBatch ab, int n_ab, int rank, int rows_per_slot, int n_ts, CurveArgs ca,
                    float* __restrict__ mods, long long mods_stride, const float* __restrict__ pos, int n,
                    InvFreq inv, float2* __restrict__ cs) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ __align__(16) float part[8][32 * 8];
  __shared__ __align__(16) float coord[8][32];
  __shared__ float sinv[K > 0 ? K : 1];
  if constexpr (K > 0) {
    if (threadIdx.x == 0) {
#pragma unroll
      for (int i = 0; i < K; ++i) sinv[i] = inv.v[i];  // static indices: no local copy of the parameter
    }
    __syncthreads();
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nq = rank >> 2;
  const int row_items = (n_ts * rows_per_slot) >> 5;  // per block
  const int ad_items = n_ab * row_items;              // < 2^31 (checked by the host)
  const int n_warps = gridDim.x * 8;
  const int gw = blockIdx.x * 8 + warp;
  float* pw = part[warp];
  float* cw = coord[warp];
  // adaLN: each warp walks its own contiguous range of items, so the curve
  // coordinates (one block, one slot) are recomputed only where the range
  // crosses a slot, and consecutive items read consecutive basis rows.
  const int chunk = (ad_items + n_warps - 1) / n_warps;
  const int it_end = min(ad_items, (gw + 1) * chunk);
  int cur = -1;  // bb * 2 + slot of the coordinates in cw
  for (int it = gw * chunk; it < it_end; ++it) {
    const int bb = it / row_items;
    const int row0 = (it - bb * row_items) << 5;
    const float4* w4 = reinterpret_cast<const float4*>(ab.w[bb] + (size_t)row0 * rank);
    float4 v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q)
      if (q < nq) v[q] = __ldcs(w4 + lane + 32 * q);
    const float bias = __ldg(ab.b[bb] + row0 + lane);
    const int sl = row0 / rows_per_slot;
    if (bb * 2 + sl != cur) {
      cur = bb * 2 + sl;
      __syncwarp();
      if (lane < rank) {
        const float* tb = ab.table[bb];
        const float a = __ldg(tb + ca.i0[sl] * rank + lane);
        const float b2 = __ldg(tb + (ca.i0[sl] + 1) * rank + lane);
        cw[lane] = (1.0f - ca.f[sl]) * a + ca.f[sl] * b2;
      }
      __syncwarp();
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (q < nq) {
        const int idx = lane + 32 * q;
        const float4 c = *reinterpret_cast<const float4*>(cw + 4 * (idx % nq));
        pw[idx] = fmaf(v[q].w, c.w, fmaf(v[q].z, c.z, fmaf(v[q].y, c.y, v[q].x * c.x)));
      }
    }
    __syncwarp();
    float acc = 0.f;
    for (int q = 0; q < nq; ++q) acc += pw[lane * nq + q];
    __stcs(mods + bb * mods_stride + row0 + lane, acc + bias);
    __syncwarp();
  }
  if constexpr (K > 0) {
    // rotation table, frequency-major: entry e = j * n + i holds pair j of
    // row i, so a warp writes (and the qkv epilogue, one row per lane, later
    // reads) 32 consecutive rows of one pair as one contiguous run.  256
    // entries per warp item, grid-stride.
    const unsigned cs_total = (unsigned)n * 3u * K;  // < 2^31 (checked by the host)
    for (unsigned e0 = (unsigned)gw * 256u; e0 < cs_total; e0 += (unsigned)n_warps * 256u) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const unsigned e = e0 + u * 32 + lane;
        if (e < cs_total) {
          const unsigned j = e / (unsigned)n, i = e - j * (unsigned)n;
          const float a = (float)((double)pos[i * 3 + j / K] * (double)sinv[j % K]);
          float sv, cv;
          sincosf(a, &sv, &cv);
          cs[e] = make_float2(cv, sv);
        }
      }
    }
  }
}

// The adaLN rows of ab's first n_ab blocks into mods + b * mods_stride
// (floats) and, when pos != null, the rotation table of n rows into cs.
// The fast path needs rank % 4 == 0 (16-byte basis rows) and
// rows_per_slot % 32 == 0; other shapes run the per-row adaln_kernel once
// per block, and the table alone through the prologue kernel.
cudaError_t launch_prologue(const AdalnBatch& ab, int n_ab, int rank, int grid, int rows_per_slot,
                            const Plan& plan, float* mods, long long mods_stride, const float* pos, int n,
                            int k, float theta, float2* cs, cudaStream_t s) {
  CurveArgs ca{};
  for (int i = 0; i < plan.n_ts; ++i) curve_coords(plan.ts[i], grid, &ca.i0[i], &ca.f[i]);
  if (n_ab < 0 || n_ab > kAdalnBatch || (pos != nullptr && (long long)n * 3 * k >= (1ll << 31)) ||
      (long long)n_ab * plan.n_ts * rows_per_slot >= (1ll << 31))
    return cudaErrorInvalidValue;
  bool fast = rank % 4 == 0 && rank <= 32 && rows_per_slot % 32 == 0;
  for (int i = 0; i < n_ab && fast; ++i)
    if (reinterpret_cast<uintptr_t>(ab.w[i]) & 15) fast = false;
  if (!fast) {
    for (int i = 0; i < n_ab; ++i) {
      const int total = plan.n_ts * rows_per_slot;
      int blocks = (total + 255) / 256;
      if (blocks > num_sms() * 8) blocks = num_sms() * 8;
      adaln_kernel<<<blocks, 256, 0, s>>>(ab.w[i], ab.b[i], ab.table[i], rank, rows_per_slot, plan.n_ts, ca,
                                          mods + i * mods_stride);
      count_launch();
      cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    n_ab = 0;
  }
  InvFreq inv{};
  for (int i = 0; i < k && i < 32; ++i) inv.v[i] = (float)std::pow((double)theta, -(double)i / (double)k);
  const int kk = pos ? k : 0;
  const long long items = (long long)n_ab * ((long long)plan.n_ts * rows_per_slot / 32) +
                          ((long long)n * 3 * kk + 255) / 256;
  if (items == 0) return cudaSuccess;
  long long blocks = (items + 7) / 8;
  if (blocks > (long long)num_sms() * 4) blocks = (long long)num_sms() * 4;  // 32 warps per SM
  const int g = (int)blocks;
  cudaError_t e;
  if (kk == 16)
    e = launch_pdl(prologue_kernel<16>, dim3(g), dim3(256), 0, s, ab, n_ab, rank, rows_per_slot, plan.n_ts, ca, mods,
                   mods_stride, pos, n, inv, cs);
  else if (kk == 8)
    e = launch_pdl(prologue_kernel<8>, dim3(g), dim3(256), 0, s, ab, n_ab, rank, rows_per_slot, plan.n_ts, ca, mods,
                   mods_stride, pos, n, inv, cs);
  else if (kk == 0)
    e = launch_pdl(prologue_kernel<0>, dim3(g), dim3(256), 0, s, ab, n_ab, rank, rows_per_slot, plan.n_ts, ca, mods,
                   mods_stride, pos, n, inv, cs);
  else
    return cudaErrorInvalidValue;
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_adaln(const float* w, const float* b, const float* table, int rank, int grid,
                         int rows_per_slot, const Plan& plan, float* out, cudaStream_t s) {
  AdalnBatch ab{};
  ab.w[0] = w;
  ab.b[0] = b;
  ab.table[0] = table;
  return launch_prologue(ab, 1, rank, grid, rows_per_slot, plan, out, 0, nullptr, 0, 0, 0.f, nullptr, s);
}

// ------------------------------------------- K2 RMSNorm + modulate gather
// y = (x * rsqrt(mean x^2 + eps) * g) * (1 + scale) + shift for each token
// row i, with shift / scale from modulation row seg_row(i + row_base),
// stored as the GEMM operand dtype.  H = 128 * VPL (VPL float4 per lane).
//
// Persistent and streaming: warp w of the grid takes rows w, w + W, ...
// (W warps in all).  Each warp owns kNormStages row buffers in shared memory;
// its lane 0 fetches rows into them with 1-D bulk copies (evict-first in L2,
// so the normalised output, which the next GEMM reads, stays there longer).
// A warp copies the current row from shared memory into registers, hands
// the buffer to the copy kNormStages rows ahead and normalises from
// registers, so two rows per warp are in flight while it computes.
constexpr int kNormStages = 2;
constexpr size_t kNormSmemBudget = 220 * 1024;
constexpr int kNormMaxWarps = 8;

__device__ __forceinline__ void store4(__nv_bfloat16* p, float4 v) {
  uint2 u;
  u.x = pack_bf16x2(v.x, v.y);
  u.y = pack_bf16x2(v.z, v.w);
  *reinterpret_cast<uint2*>(p) = u;
}
__device__ __forceinline__ void store4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }

template <typename TO, int VPL>
__global__ void __launch_bounds__(kNormMaxWarps * 32, 1)
    norm_mod_kernel(const float* __restrict__ x, int n, int H, const float* __restrict__ g, float eps,
                    const float* __restrict__ mods, int mods_stride, int shift_off, int scale_off, SegRows seg,
                    int row_base, TO* __restrict__ out, unsigned* zero_word, DevStatus* status,
                    uint64_t limit_ns) {
  pdl_launch_dependents();
  pdl_wait();
  if (zero_word != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *zero_word = 0u;
  constexpr uint32_t kRowBytes = VPL * 512;
  extern __shared__ __align__(128) uint8_t norm_smem[];
  const int warps = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float4* buf = reinterpret_cast<const float4*>(norm_smem + (size_t)warp * kNormStages * kRowBytes);
  const uint32_t buf_s = smem_u32(buf);
  const uint32_t bar0 = smem_u32(norm_smem + (size_t)warps * kNormStages * kRowBytes) + 8u * kNormStages * warp;
  const long long W = (long long)gridDim.x * warps;
  const long long gw = (long long)blockIdx.x * warps + warp;
  const int cnt = gw < n ? (int)((n - 1 - gw) / W) + 1 : 0;  // rows of this warp
  if (cnt == 0) return;  // warp-uniform; the kernel has no CTA-wide barrier
  uint64_t policy = 0;
  if (lane == 0) {
    for (int st = 0; st < kNormStages; ++st) mbar_init(bar0 + 8u * st, 1);
    fence_mbar_init();
    policy = policy_evict_first();
  }
  __syncwarp();
  auto issue = [&](int i) {  // lane 0: row i of this warp into buffer i % kNormStages
    const uint32_t st = (uint32_t)(i % kNormStages);
    mbar_expect_tx(bar0 + 8u * st, kRowBytes);
    bulk_load_1d(buf_s + st * kRowBytes, x + (size_t)(gw + (long long)i * W) * H, kRowBytes, bar0 + 8u * st,
                 policy);
  };
  if (lane == 0)
    for (int i = 0; i < kNormStages && i < cnt; ++i) issue(i);
  const float4* g4 = reinterpret_cast<const float4*>(g);
  int i = 0;
  for (; i < cnt; ++i) {
    const int st = i % kNormStages;
    const bool fail = !mbar_wait(bar0 + 8u * st, (uint32_t)((i / kNormStages) & 1), limit_ns);
    if (__any_sync(0xffffffffu, fail)) break;
    float4 v[VPL];
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < VPL; ++k) v[k] = buf[st * (VPL * 32) + k * 32 + lane];
    // every lane holds its part of the row: the buffer takes the next copy
    // (the proxy fence orders these reads before the copy's writes)
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && i + kNormStages < cnt) issue(i + kNormStages);
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      ss = fmaf(v[k].x, v[k].x, ss);
      ss = fmaf(v[k].y, v[k].y, ss);
      ss = fmaf(v[k].z, v[k].z, ss);
      ss = fmaf(v[k].w, v[k].w, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = rsqrtf(ss / (float)H + eps);
    const int row = (int)(gw + (long long)i * W);
    const float* m = mods ? mods + (size_t)seg_row_checked(seg, row + row_base) * mods_stride : nullptr;
    TO* o = out + (size_t)row * H;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      const int c4 = k * 32 + lane;
      const float4 gg = __ldg(g4 + c4);
      float4 y = make_float4(v[k].x * inv * gg.x, v[k].y * inv * gg.y, v[k].z * inv * gg.z,
                             v[k].w * inv * gg.w);
      if (m) {
        const float4 sh = __ldg(reinterpret_cast<const float4*>(m + shift_off) + c4);
        const float4 sc = __ldg(reinterpret_cast<const float4*>(m + scale_off) + c4);
        y.x = fmaf(y.x, 1.0f + sc.x, sh.x);
        y.y = fmaf(y.y, 1.0f + sc.y, sh.y);
        y.z = fmaf(y.z, 1.0f + sc.z, sh.z);
        y.w = fmaf(y.w, 1.0f + sc.w, sh.w);
      }
      store4(o + 4 * c4, y);
    }
  }
  if (i < cnt && lane == 0) {
    // gave up on row i: record it, then let the copies still in flight land
    // (bounded) before the CTA's shared memory is released
    record_error(status, DEV_TIMEOUT_COPY, (int)(gw + (long long)i * W));
    for (int k = i; k < cnt && k < i + kNormStages; ++k)
      mbar_wait(bar0 + 8u * (uint32_t)(k % kNormStages), (uint32_t)((k / kNormStages) & 1), limit_ns);
  }
}

// Warps per CTA: as many as the row buffers' shared memory allows (at most
// kNormMaxWarps; more warps would cap a thread's registers at 168 and
// spill), fewer only where that leaves a fuller last round of rows (e.g.
// 13 248 rows on 148 SMs: seven warps a CTA give 13 rounds, 98% full,
// against 12 rounds, 93% full, with eight).
template <typename TO, int VPL>
static cudaError_t norm_mod_launch(const float* x, int n, int H, const float* g, float eps, const float* mods,
                                   int ms, int so, int co, const SegRows& seg, int rb, TO* out, cudaStream_t s,
                                   unsigned* zw) {
  constexpr size_t kWarpBytes = (size_t)kNormStages * (VPL * 512 + 8);
  constexpr int kWarps = kNormSmemBudget / kWarpBytes >= kNormMaxWarps ? kNormMaxWarps
                                                                         : (int)(kNormSmemBudget / kWarpBytes);
  static_assert(kWarps >= 1, "RMSNorm row buffers above the shared-memory budget");
  auto kern = norm_mod_kernel<TO, VPL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)(kWarps * kWarpBytes));
  if (e != cudaSuccess) return e;
  static int per_sm[64][kNormMaxWarps + 1];  // CTAs per SM by warps per CTA (0: not yet asked)
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  const long long sms = num_sms();
  int warps = kWarps, ctas_per_sm = 1;
  double best = -1.0;
  for (int w = kWarps; w >= 1 && w >= kWarps - 4; --w) {
    if (per_sm[dev][w] == 0) {
      int v = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, kern, w * 32, w * kWarpBytes);
      if (e != cudaSuccess) return e;
      per_sm[dev][w] = v > 0 ? v : 1;
    }
    const long long lanes = sms * per_sm[dev][w] * w;  // warps resident at once
    const long long rounds = ((long long)n + lanes - 1) / lanes;
    const double full = (double)n / (double)(rounds * lanes);
    if (full > best + 0.02) {
      best = full;
      warps = w;
      ctas_per_sm = per_sm[dev][w];
    }
    if (rounds == 1) break;  // one round: fewer warps a CTA only spread the same rows thinner
  }
  const long long want = ((long long)n + warps - 1) / warps;
  const long long cap = sms * ctas_per_sm;
  const int blocks = (int)(want < cap ? want : cap);
  e = launch_pdl(kern, dim3(blocks), dim3(warps * 32), warps * kWarpBytes, s, x, n, H, g, eps, mods, ms, so, co, seg,
                 rb, out, zw, device_status_ptr(), wait_limit_ns());
  count_launch();
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename TO>
static cudaError_t norm_mod_dispatch(const float* x, int n, int H, const float* g, float eps,
                                     const float* mods, int ms, int so, int co, const SegRows& seg,
                                     int rb, TO* out, cudaStream_t s, unsigned* zw) {
  switch (H / 128) {
#define MMH3_NM(V) \
  case V:          \
    return norm_mod_launch<TO, V>(x, n, H, g, eps, mods, ms, so, co, seg, rb, out, s, zw);
    MMH3_NM(1) MMH3_NM(2) MMH3_NM(4) MMH3_NM(6) MMH3_NM(8) MMH3_NM(16) MMH3_NM(21) MMH3_NM(24)
    MMH3_NM(32)
#undef MMH3_NM
    default:
      return cudaErrorInvalidValue;
  }
}

cudaError_t launch_norm_mod(int dtype, const float* x, int n, int H, const float* g, float eps,
                            const float* mods, int mods_stride, int shift_off, int scale_off,
                            const SegRows& seg, int row_base, void* out, cudaStream_t s, unsigned* zero_word) {
  if (n <= 0) return cudaSuccess;
  if (dtype == MMH3_BF16)
    return norm_mod_dispatch(x, n, H, g, eps, mods, mods_stride, shift_off, scale_off, seg, row_base,
                             static_cast<__nv_bfloat16*>(out), s, zero_word);
  return norm_mod_dispatch(x, n, H, g, eps, mods, mods_stride, shift_off, scale_off, seg, row_base,
                           static_cast<float*>(out), s, zero_word);
}

// ------------------------------------------------------------ LayerNorm
// One warp per row, two-pass variance over registers.
template <int VPL>
__global__ void __launch_bounds__(256) layernorm_kernel(const float* __restrict__ x, int n, int H,
                                                        const float* __restrict__ g,
                                                        const float* __restrict__ b, float eps,
                                                        __nv_bfloat16* __restrict__ out, unsigned* zero_word) {
  if (zero_word != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *zero_word = 0u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= n) return;
  const float4* xr = reinterpret_cast<const float4*>(x + (size_t)row * H);
  float4 v[VPL];
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    v[i] = __ldcs(xr + i * 32 + lane);
    sum += (v[i].x + v[i].y) + (v[i].z + v[i].w);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float mu = sum / (float)H;
  float sq = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    v[i].x -= mu; v[i].y -= mu; v[i].z -= mu; v[i].w -= mu;
    sq = fmaf(v[i].x, v[i].x, sq);
    sq = fmaf(v[i].y, v[i].y, sq);
    sq = fmaf(v[i].z, v[i].z, sq);
    sq = fmaf(v[i].w, v[i].w, sq);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  const float inv = rsqrtf(sq / (float)H + eps);
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int c4 = i * 32 + lane;
    const float4 gg = __ldg(reinterpret_cast<const float4*>(g) + c4);
    const float4 bb = __ldg(reinterpret_cast<const float4*>(b) + c4);
    const float4 y = make_float4(fmaf(v[i].x * inv, gg.x, bb.x), fmaf(v[i].y * inv, gg.y, bb.y),
                                 fmaf(v[i].z * inv, gg.z, bb.z), fmaf(v[i].w * inv, gg.w, bb.w));
    store4(out + (size_t)row * H + 4 * c4, y);
  }
}

cudaError_t launch_layernorm(const float* x, int n, int H, const float* g, const float* b,
                             float eps, __nv_bfloat16* out, cudaStream_t s, unsigned* zero_word) {
  if (n <= 0) return cudaSuccess;
  const int blocks = (n + 7) / 8;
  switch (H / 128) {
#define MMH3_LN(V) \
  case V: layernorm_kernel<V><<<blocks, 256, 0, s>>>(x, n, H, g, b, eps, out, zero_word); count_launch(); break;
    MMH3_LN(2) MMH3_LN(4) MMH3_LN(6) MMH3_LN(8) MMH3_LN(16) MMH3_LN(21)
#undef MMH3_LN
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------ row table
__global__ void rows_kernel(SegRows seg, int n, int32_t* __restrict__ rows) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    rows[i] = seg_row(seg, i);
}

cudaError_t launch_rows(const SegRows& seg, int n, int32_t* rows, cudaStream_t s) {
  int blocks = (n + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  rows_kernel<<<blocks, 256, 0, s>>>(seg, n, rows); count_launch();
  return cudaGetLastError();
}

// ------------------------------------------------- fc1 tile interleave
// out row (t*256 + j) = gate row (t*128 + j) for j < 128, else up row
// (F + t*128 + j - 128); rows of `row_bytes` bytes copied as 16-byte words.
__global__ void fc1_tile_kernel(const uint4* __restrict__ in, uint4* __restrict__ out, int F,
                                int words_per_row) {
  const long total = 2L * F * words_per_row;
  for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < total; e += (long)gridDim.x * blockDim.x) {
    const int orow = (int)(e / words_per_row), w = (int)(e % words_per_row);
    const int t = orow / 256, j = orow % 256;
    const int irow = j < 128 ? t * 128 + j : F + t * 128 + (j - 128);
    out[e] = in[(long)irow * words_per_row + w];
  }
}

cudaError_t launch_fc1_tile(int esize, const void* in, void* out, int F, int H, cudaStream_t s) {
  const int words = H * esize / 16;
  long total = 2L * F * words;
  long blocks = (total + 255) / 256;
  if (blocks > num_sms() * 32) blocks = num_sms() * 32;
  fc1_tile_kernel<<<(int)blocks, 256, 0, s>>>(static_cast<const uint4*>(in), static_cast<uint4*>(out), F,
                                              words); count_launch();
  return cudaGetLastError();
}

// -------------------------------------------------- encoder qkv folding
__global__ void vit_fold_kernel(const __nv_bfloat16* __restrict__ wq, const __nv_bfloat16* __restrict__ wk,
                                const __nv_bfloat16* __restrict__ wv, const float* __restrict__ bq,
                                const float* __restrict__ bk, const float* __restrict__ bv, float scale,
                                int H, __nv_bfloat16* __restrict__ wqkv, float* __restrict__ bqkv) {
  const long hh = (long)H * H;
  for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < 3 * hh; e += (long)gridDim.x * blockDim.x) {
    const int part = (int)(e / hh);
    const long off = e % hh;
    float v = __bfloat162float(part == 0 ? wq[off] : part == 1 ? wk[off] : wv[off]);
    if (part == 0) v *= scale;
    wqkv[e] = __float2bfloat16_rn(v);
    if (off < H) {
      const float bb = part == 0 ? bq[off] * scale : part == 1 ? bk[off] : bv[off];
      bqkv[part * H + off] = bb;
    }
  }
}

cudaError_t launch_vit_fold(const void* wq, const void* wk, const void* wv, const float* bq,
                            const float* bk, const float* bv, float scale, int H, void* wqkv,
                            float* bqkv, cudaStream_t s) {
  long total = 3L * H * H;
  long blocks = (total + 255) / 256;
  if (blocks > num_sms() * 32) blocks = num_sms() * 32;
  vit_fold_kernel<<<(int)blocks, 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(wq), static_cast<const __nv_bfloat16*>(wk),
      static_cast<const __nv_bfloat16*>(wv), bq, bk, bv, scale, H, static_cast<__nv_bfloat16*>(wqkv), bqkv); count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------- stream (un)packing
// patchify: rows[(t*(H/2) + hi)*(W/2) + wi][c*4 + p*2 + q] = x[c][t][2hi+p][2wi+q]
// (2x2 spatial patches, channel-major inside a row); pack audio:
// rows[ch*T + t][c] = x[c][ch][t] (stereo channel 0's frames, then channel 1's).
template <typename TO>
__global__ void patchify_kernel(const float* __restrict__ x, int C, int T, int H, int W, TO* __restrict__ rows) {
  const int hh = H / 2, ww = W / 2;
  const long total = (long)T * hh * ww * 4 * C;
  for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < total; e += (long)gridDim.x * blockDim.x) {
    const int col = (int)(e % (4 * C));
    const long r = e / (4 * C);
    const int wi = (int)(r % ww), hi = (int)((r / ww) % hh), t = (int)(r / ((long)ww * hh));
    const int c = col >> 2, p = (col >> 1) & 1, q = col & 1;
    const float v = x[(((long)c * T + t) * H + 2 * hi + p) * W + 2 * wi + q];
    if constexpr (sizeof(TO) == 2) rows[e] = __float2bfloat16_rn(v);
    else rows[e] = v;
  }
}

__global__ void unpatchify_kernel(const float* __restrict__ rows, int C, int T, int H, int W, float* __restrict__ x) {
  const int hh = H / 2, ww = W / 2;
  const long total = (long)T * hh * ww * 4 * C;
  for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < total; e += (long)gridDim.x * blockDim.x) {
    const int col = (int)(e % (4 * C));
    const long r = e / (4 * C);
    const int wi = (int)(r % ww), hi = (int)((r / ww) % hh), t = (int)(r / ((long)ww * hh));
    const int c = col >> 2, p = (col >> 1) & 1, q = col & 1;
    x[(((long)c * T + t) * H + 2 * hi + p) * W + 2 * wi + q] = rows[e];
  }
}

template <typename TO>
__global__ void pack_audio_kernel(const float* __restrict__ x, int C, int T, TO* __restrict__ rows) {
  const long total = 2L * T * C;
  for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < total; e += (long)gridDim.x * blockDim.x) {
    const int c = (int)(e % C);
    const long r = e / C;
    const int ch = (int)(r / T), t = (int)(r % T);
    const float v = x[((long)c * 2 + ch) * T + t];
    if constexpr (sizeof(TO) == 2) rows[e] = __float2bfloat16_rn(v);
    else rows[e] = v;
  }
}

__global__ void unpack_audio_kernel(const float* __restrict__ rows, int C, int T, float* __restrict__ x) {
  const long total = 2L * T * C;
  for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < total; e += (long)gridDim.x * blockDim.x) {
    const int c = (int)(e % C);
    const long r = e / C;
    const int ch = (int)(r / T), t = (int)(r % T);
    x[((long)c * 2 + ch) * T + t] = rows[e];
  }
}

static int grid_for(long total) {
  long b = (total + 255) / 256;
  const long cap = (long)num_sms() * 16;
  return (int)(b < 1 ? 1 : (b > cap ? cap : b));
}

cudaError_t launch_patchify(int dtype, const float* x, int C, int T, int H, int W, void* rows, cudaStream_t s) {
  const long total = (long)T * (H / 2) * (W / 2) * 4 * C;
  if (dtype == MMH3_BF16)
    patchify_kernel<__nv_bfloat16><<<grid_for(total), 256, 0, s>>>(x, C, T, H, W, static_cast<__nv_bfloat16*>(rows));
  else
    patchify_kernel<float><<<grid_for(total), 256, 0, s>>>(x, C, T, H, W, static_cast<float*>(rows));
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_unpatchify(const float* rows, int C, int T, int H, int W, float* x, cudaStream_t s) {
  unpatchify_kernel<<<grid_for((long)T * (H / 2) * (W / 2) * 4 * C), 256, 0, s>>>(rows, C, T, H, W, x); count_launch();
  return cudaGetLastError();
}

cudaError_t launch_pack_audio(int dtype, const float* x, int C, int T, void* rows, cudaStream_t s) {
  const long total = 2L * T * C;
  if (dtype == MMH3_BF16)
    pack_audio_kernel<__nv_bfloat16><<<grid_for(total), 256, 0, s>>>(x, C, T, static_cast<__nv_bfloat16*>(rows));
  else
    pack_audio_kernel<float><<<grid_for(total), 256, 0, s>>>(x, C, T, static_cast<float*>(rows));
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_unpack_audio(const float* rows, int C, int T, float* x, cudaStream_t s) {
  unpack_audio_kernel<<<grid_for(2L * T * C), 256, 0, s>>>(rows, C, T, x); count_launch();
  return cudaGetLastError();
}

// ------------------------------------------------ bounded-wait self test
// One thread initialises an mbarrier that expects one arrival which never
// comes, waits with the given limit and records the timeout.
__global__ void selftest_wait_kernel(uint64_t limit_ns, DevStatus* st) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    const uint32_t b = smem_u32(&bar);
    mbar_init(b, 1);
    fence_mbar_init();
    if (!mbar_wait(b, 0, limit_ns)) record_error(st, DEV_TIMEOUT_SELFTEST, 0);
  }
}

cudaError_t launch_selftest_wait(uint64_t limit_ns, cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(limit_ns, device_status_ptr()); count_launch();
  return cudaGetLastError();
}

}  // namespace mmh3

using namespace mmh3;

extern "C" mmh3_status mmh3_device_status(void* stream, int* code, int* site) {
  clear_error();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "device_status: stream synchronize");
  DevStatus* p = device_status_ptr();
  if (p == nullptr) return fail(MMH3_ERR_CUDA, "device_status: no status symbol");
  DevStatus h{};
  e = cudaMemcpy(&h, p, sizeof(h), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "device_status: read");
  const int zero[3] = {0, 0, 0};  // code, site, count; the check flag stays
  e = cudaMemcpy(p, zero, sizeof(zero), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "device_status: clear");
  if (code) *code = h.code;
  if (site) *site = h.site;
  if (dev_err_is_check(h.code))
    return fail(MMH3_ERR_CHECK, "a device check failed (code %d, site %d, %d records)", h.code, h.site, h.count);
  if (h.code != 0)
    return fail(MMH3_ERR_TIMEOUT, "a kernel gave up waiting (code %d, site %d, %d CTAs)", h.code, h.site,
                h.count);
  return MMH3_OK;
}

extern "C" mmh3_status mmh3_status_sync(void* stream, int* device_status) {
  return mmh3_device_status(stream, device_status, nullptr);
}

extern "C" mmh3_status mmh3_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
  clear_error();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_selftest_wait(limit_ns, s);
  if (e != cudaSuccess) return cuda_fail(e, "selftest launch");
  int code = 0, site = 0;
  return mmh3_device_status(stream, &code, &site);
}
