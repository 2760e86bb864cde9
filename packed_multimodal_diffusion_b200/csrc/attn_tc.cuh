// Bidirectional flash attention on tcgen05 for the packed sequence.
//
// One CTA computes one 128-row query tile of one head:
//   warp 0      TMA producer: Q once, then K_j and V_j tiles (double buffered)
//   warp 1      MMA issuer: S_j = Q K_j^T into TMEM (two S buffers), then
//               O += P_j V_j into a TMEM accumulator once P_j is written
//   warps 2..5  softmax: thread r owns query row r; reads S_j from TMEM,
//               keeps a running row maximum and sum in the log2 domain,
//               writes P_j = 2^(s*scale*log2e - m) into swizzled shared
//               memory (the MMA's A operand), rescales O in TMEM only when
//               the maximum grows by more than 2^8 (the final division by
//               the row sum uses the same reference maximum, so a stale
//               maximum is exact up to rounding), and in the end divides O
//               by the row sum and stores it (late normalisation).
// K and V tiles are read from the qkv panel [rows, 3*inner] in place by TMA
// boxes of 128 rows x 128 bytes; the V operand is MN-major.  Sequences are
// `seq` tokens long and start at blockIdx.z * seq (independent images for
// the encoder layer; one sequence for the packed DiT).  Keys at or beyond the
// sequence end are masked; query rows beyond it are not stored.
#pragma once

#include "gemm_tc.cuh"

namespace mmh3 {

template <typename T, int HD, int KV_STAGES, int P_BUFS>
struct AttnShape {
  static constexpr int kEB = ElemTraits<T>::kBytes;
  static constexpr int kEPB = 128 / kEB;          // elements per 128-byte box row
  static constexpr int kUK = 32 / kEB;            // K elements per MMA instruction
  static constexpr int kBoxBytes = 128 * 128;     // 128 rows x 128 bytes
  static constexpr int kHdBoxes = HD / kEPB;      // boxes across a head
  static constexpr int kTileBytes = kHdBoxes * kBoxBytes;
  static constexpr int kPBoxes = 128 / kEPB;      // boxes across 128 keys
  static constexpr int kPBytes = kPBoxes * kBoxBytes;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kTileBytes;
  static constexpr int kVOff = kKOff + KV_STAGES * kTileBytes;
  static constexpr int kPOff = kVOff + KV_STAGES * kTileBytes;
  static constexpr int kBarOff = kPOff + P_BUFS * kPBytes;
  static constexpr int kSmem = kBarOff + 512 + 1024;
  static constexpr int kTmemCols = 512;  // S0 @0, S1 @128, O @256
};

template <typename T, int HD, int KV_STAGES, int P_BUFS>
__global__ void __launch_bounds__(192, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm, T* __restrict__ out, int ldo, int seq,
                   int inner, float scale_log2, DevStatus* status, uint64_t limit_ns) {
  using Sh = AttnShape<T, HD, KV_STAGES, P_BUFS>;
  constexpr bool kTf32 = ElemTraits<T>::kTf32;
  constexpr uint32_t kIdescS = make_idesc(kTf32, 128, 128, false, false);
  constexpr uint32_t kIdescO = make_idesc(kTf32, 128, HD, false, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Sh::kBarOff);
  // barrier indices
  constexpr int B_Q = 0;
  constexpr int B_KF = 1, B_KE = B_KF + KV_STAGES, B_VF = B_KE + KV_STAGES, B_VE = B_VF + KV_STAGES;
  constexpr int B_SF = B_VE + KV_STAGES, B_SE = B_SF + 2, B_PF = B_SE + 2, B_PV = B_PF + P_BUFS;
  constexpr int B_DRAIN = B_PV + P_BUFS;
  constexpr int kNumBars = B_DRAIN + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = smem_u32(bars);
  auto bar = [&](int i) { return bar0 + 8u * i; };

  const int qt = blockIdx.x, head = blockIdx.y;
  const int seq_row0 = blockIdx.z * seq;
  const int q_row0 = seq_row0 + qt * 128;
  const int n_kv = (seq + 127) / 128;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_Q), 1);
    for (int s = 0; s < KV_STAGES; ++s) {
      mbar_init(bar(B_KF + s), 1);
      mbar_init(bar(B_KE + s), 1);
      mbar_init(bar(B_VF + s), 1);
      mbar_init(bar(B_VE + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_SF + s), 1);
      mbar_init(bar(B_SE + s), 128);
    }
    for (int s = 0; s < P_BUFS; ++s) {
      mbar_init(bar(B_PF + s), 128);
      mbar_init(bar(B_PV + s), 1);
    }
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch(&tm);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), Sh::kTmemCols);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_o = tmem + 256;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      const int xq = head * HD, xk = inner + head * HD, xv = 2 * inner + head * HD;
      int in_flight_k = 0, in_flight_v = 0;
      bool ok = true;
      mbar_expect_tx(bar(B_Q), Sh::kTileBytes);
      for (int c = 0; c < Sh::kHdBoxes; ++c)
        tma_load_2d(sbase + Sh::kQOff + c * Sh::kBoxBytes, &tm, bar(B_Q), xq + c * Sh::kEPB, q_row0);
      int j = 0;
      for (; j < n_kv && ok; ++j) {
        const int s = j % KV_STAGES;
        const uint32_t ph = (uint32_t)((j / KV_STAGES) & 1);
        const int y = seq_row0 + j * 128;
        if (*abort_flag || !mbar_wait(bar(B_KE + s), ph ^ 1u, limit_ns)) { ok = false; break; }
        mbar_expect_tx(bar(B_KF + s), Sh::kTileBytes);
        for (int c = 0; c < Sh::kHdBoxes; ++c)
          tma_load_2d(sbase + Sh::kKOff + s * Sh::kTileBytes + c * Sh::kBoxBytes, &tm, bar(B_KF + s),
                      xk + c * Sh::kEPB, y);
        in_flight_k = j + 1;
        if (*abort_flag || !mbar_wait(bar(B_VE + s), ph ^ 1u, limit_ns)) { ok = false; break; }
        mbar_expect_tx(bar(B_VF + s), Sh::kTileBytes);
        for (int c = 0; c < Sh::kHdBoxes; ++c)
          tma_load_2d(sbase + Sh::kVOff + s * Sh::kTileBytes + c * Sh::kBoxBytes, &tm, bar(B_VF + s),
                      xv + c * Sh::kEPB, y);
        in_flight_v = j + 1;
      }
      if (!ok) {
        if (!*abort_flag) record_error(status, DEV_TIMEOUT_PRODUCER, j);
        *abort_flag = 1;
        // drain the copies that may still be landing
        mbar_wait(bar(B_Q), 0, limit_ns);
        for (int i = (in_flight_k > KV_STAGES ? in_flight_k - KV_STAGES : 0); i < in_flight_k; ++i)
          mbar_wait(bar(B_KF + i % KV_STAGES), (uint32_t)((i / KV_STAGES) & 1), limit_ns);
        for (int i = (in_flight_v > KV_STAGES ? in_flight_v - KV_STAGES : 0); i < in_flight_v; ++i)
          mbar_wait(bar(B_VF + i % KV_STAGES), (uint32_t)((i / KV_STAGES) & 1), limit_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      bool ok = mbar_wait(bar(B_Q), 0, limit_ns);
      auto issue_pv = [&](int i) -> bool {
        const int s = i % KV_STAGES, pb = i % P_BUFS;
        if (*abort_flag || !mbar_wait(bar(B_PF + pb), (uint32_t)((i / P_BUFS) & 1), limit_ns)) return false;
        if (*abort_flag || !mbar_wait(bar(B_VF + s), (uint32_t)((i / KV_STAGES) & 1), limit_ns)) return false;
        tc_fence_after();
        const uint32_t pa = sbase + Sh::kPOff + pb * Sh::kPBytes;
        const uint32_t va = sbase + Sh::kVOff + s * Sh::kTileBytes;
#pragma unroll
        for (int ks = 0; ks < 128 / Sh::kUK; ++ks) {
          const uint64_t ad = sdesc_sw128(pa + (ks / 4) * Sh::kBoxBytes + (ks % 4) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(va + ks * Sh::kUK * 128, Sh::kBoxBytes, 1024);
          umma_ss<kTf32>(t_o, ad, bd, kIdescO, (i > 0 || ks > 0) ? 1u : 0u);
        }
        umma_commit(bar(B_VE + s));
        umma_commit(bar(B_PV + pb));
        return true;
      };
      for (int j = 0; j < n_kv && ok; ++j) {
        const int s = j % KV_STAGES, sb = j & 1;
        if (*abort_flag || !mbar_wait(bar(B_KF + s), (uint32_t)((j / KV_STAGES) & 1), limit_ns)) { ok = false; break; }
        if (j >= 2 && (*abort_flag || !mbar_wait(bar(B_SE + sb), (uint32_t)(((j - 2) / 2) & 1), limit_ns))) { ok = false; break; }
        tc_fence_after();
        const uint32_t ka = sbase + Sh::kKOff + s * Sh::kTileBytes;
        const uint32_t qa = sbase + Sh::kQOff;
#pragma unroll
        for (int ks = 0; ks < HD / Sh::kUK; ++ks) {
          const uint32_t off = (ks / 4) * Sh::kBoxBytes + (ks % 4) * 32;
          umma_ss<kTf32>(tmem + sb * 128, sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(ka + off, 16, 1024),
                         kIdescS, ks > 0 ? 1u : 0u);
        }
        umma_commit(bar(B_KE + s));
        umma_commit(bar(B_SF + sb));
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok) ok = issue_pv(n_kv - 1);
      if (!ok) {
        if (!*abort_flag) record_error(status, DEV_TIMEOUT_MMA, blockIdx.x);
        *abort_flag = 1;
        umma_commit(bar(B_DRAIN));
        mbar_wait(bar(B_DRAIN), 0, limit_ns);
      }
    }
  } else {
    // -------------------------------------------------- softmax warps
    const int lgrp = warp & 3;
    const int r = lgrp * 32 + lane;  // query row within the tile
    const uint32_t lane_off = (uint32_t)(lgrp * 32) << 16;
    float m_ref = 0.f, l_sum = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int sb = j & 1, pb = j % P_BUFS;
      {
        // warp-uniform decision: the TMEM loads below are warp-collective
        const bool fail = *abort_flag || !mbar_wait(bar(B_SF + sb), (uint32_t)((j / 2) & 1), limit_ns);
        if (__any_sync(0xffffffffu, fail)) { ok = false; break; }
      }
      tc_fence_after();
      float s[128];
      {
        // four loads in flight, one wait
        uint32_t u0[32], u1[32], u2[32], u3[32];
        const uint32_t ts = tmem + sb * 128 + lane_off;
        tmem_ld32(ts + 0, u0);
        tmem_ld32(ts + 32, u1);
        tmem_ld32(ts + 64, u2);
        tmem_ld32(ts + 96, u3);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          s[i] = __uint_as_float(u0[i]);
          s[32 + i] = __uint_as_float(u1[i]);
          s[64 + i] = __uint_as_float(u2[i]);
          s[96 + i] = __uint_as_float(u3[i]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(B_SE + sb));
      const int valid = seq - j * 128;
      if (valid < 128) {
#pragma unroll
        for (int k = 0; k < 128; ++k)
          if (k >= valid) s[k] = -INFINITY;
      }
      // row maximum with eight independent partial maxima (short chains)
      float pm[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) pm[i] = s[i];
#pragma unroll
      for (int k = 8; k < 128; ++k) pm[k & 7] = fmaxf(pm[k & 7], s[k]);
      const float mx = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                             fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
      const float m_tile = mx * scale_log2;
      if (j == 0) {
        m_ref = m_tile;
      } else {
        const bool need = m_tile > m_ref + 8.0f;
        if (__any_sync(0xffffffffu, need)) {
          // O must hold every earlier P V product before it is rescaled.
          const int i = j - 1;
          if (*abort_flag || !mbar_wait(bar(B_PV + i % P_BUFS), (uint32_t)((i / P_BUFS) & 1), limit_ns)) {
            ok = false;
          }
          if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
          tc_fence_after();
          const float m_new = need ? m_tile : m_ref;
          const float f = ex2_approx(m_ref - m_new);
          l_sum *= f;
          m_ref = m_new;
#pragma unroll 1
          for (int c = 0; c < HD / 32; ++c) {
            uint32_t u[32];
            tmem_ld32(t_o + lane_off + c * 32, u);
            tmem_wait_ld();
#pragma unroll
            for (int i2 = 0; i2 < 32; ++i2) u[i2] = __float_as_uint(__uint_as_float(u[i2]) * f);
            tmem_st32(t_o + lane_off + c * 32, u);
          }
          tmem_wait_st();
        }
      }
      // P buffer pb was last read by P V of tile j - P_BUFS.
      if (j >= P_BUFS) {
        const int i = j - P_BUFS;
        if (*abort_flag || !mbar_wait(bar(B_PV + pb), (uint32_t)((i / P_BUFS) & 1), limit_ns)) ok = false;
        if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
      }
      // p = 2^(s * scale * log2e - m_ref); write the row into the swizzled
      // K-major A tile: box = key / kEPB, 16-byte chunk index XOR (row % 8).
      uint8_t* prow = smem + Sh::kPOff + pb * Sh::kPBytes + r * 128;
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (kTf32) {
#pragma unroll
        for (int k8 = 0; k8 < 128 / 4; ++k8) {
          float4 q;
          q.x = ex2_approx(fmaf(s[4 * k8 + 0], scale_log2, -m_ref));
          q.y = ex2_approx(fmaf(s[4 * k8 + 1], scale_log2, -m_ref));
          q.z = ex2_approx(fmaf(s[4 * k8 + 2], scale_log2, -m_ref));
          q.w = ex2_approx(fmaf(s[4 * k8 + 3], scale_log2, -m_ref));
          ps[k8 & 3] += (q.x + q.y) + (q.z + q.w);
          const int box = k8 / 8, chunk = k8 % 8;
          *reinterpret_cast<float4*>(prow + box * Sh::kBoxBytes + ((chunk ^ (r & 7)) * 16)) = q;
        }
      } else {
#pragma unroll
        for (int k8 = 0; k8 < 128 / 8; ++k8) {
          float p[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) p[e] = ex2_approx(fmaf(s[8 * k8 + e], scale_log2, -m_ref));
          ps[k8 & 3] += ((p[0] + p[1]) + (p[2] + p[3])) + ((p[4] + p[5]) + (p[6] + p[7]));
          uint4 q;
          q.x = pack_bf16x2(p[0], p[1]);
          q.y = pack_bf16x2(p[2], p[3]);
          q.z = pack_bf16x2(p[4], p[5]);
          q.w = pack_bf16x2(p[6], p[7]);
          const int box = k8 / 8, chunk = k8 % 8;
          *reinterpret_cast<uint4*>(prow + box * Sh::kBoxBytes + ((chunk ^ (r & 7)) * 16)) = q;
        }
      }
      l_sum += (ps[0] + ps[1]) + (ps[2] + ps[3]);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(B_PF + pb));
    }
    if (ok) {
      const int i = n_kv - 1;
      if (*abort_flag || !mbar_wait(bar(B_PV + i % P_BUFS), (uint32_t)((i / P_BUFS) & 1), limit_ns)) ok = false;
    }
    if (!ok) {
      if (!*abort_flag) record_error(status, DEV_TIMEOUT_SOFTMAX, blockIdx.x);
      *abort_flag = 1;
    }
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      const float inv = l_sum > 0.f ? 1.0f / l_sum : 0.f;
      const bool row_ok = (qt * 128 + r) < seq;
      T* dst = out + (size_t)(q_row0 + r) * ldo + head * HD;
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        float v[32];
        ld_acc32(t_o + lane_off + c * 32, v);
#pragma unroll
        for (int i2 = 0; i2 < 32; ++i2) v[i2] *= inv;
        if (row_ok) store32(dst + c * 32, v);
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Sh::kTmemCols);
  }
}

}  // namespace mmh3
