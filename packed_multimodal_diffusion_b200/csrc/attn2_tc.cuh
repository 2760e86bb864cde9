// Bidirectional flash attention on tcgen05, two query tiles per work item.
//
// A work item is two 128-row query tiles (256 rows) of one head, over all
// its keys or one key range of them, so each K/V tile fetched by TMA serves
// 256 query rows.  Tensor memory (512 columns) holds S0 | S1 | O0 | O1.
//   warp 0      TMA producer: Q0 and Q1 of the item, then its K_j / V_j
//               (two stages)
//   warp 1      MMA issuer (the whole warp runs the loop, one elected lane
//               issues): S0 = Q0 K_0^T, S1 = Q1 K_0^T, then per key tile
//               j: O0 += P0 V_j (once P0 is written), S0 = Q0 K_{j+1}^T,
//               O1 += P1 V_j (once P1 is written), S1 = Q1 K_{j+1}^T
//               P_i (bf16) is read as the A operand straight from tensor
//               memory, where softmax warpgroup i wrote it over the first 64
//               columns of S_i.  P_i arrives in two halves of 64 keys, and
//               the first half of O_i += P_i V_j is issued as soon as the
//               softmax has released it.  MMAs of one thread run in issue order, so
//               S_i(j+1) (issued after O_i += P_i V_j) cannot overwrite P_i
//               before that product has read it; and the commit that
//               signals S_i(j+1) also covers O_i += P_i V_j, so O_i is
//               stable when softmax i sees S_i(j+1).
//   warps 2..5  softmax of tile 0, warps 6..9 softmax of tile 1: thread r
//               owns query row r; running maximum in the log2 domain, O
//               rescaled only when the maximum grows by more than 2^8 (the
//               final division uses the same reference maximum, so a stale
//               maximum is exact up to rounding); late normalisation in the
//               epilogue.  After the first key tile the exponentials are
//               computed against the current reference maximum while the
//               tile's own maximum is found; a row whose maximum outgrew the
//               reference by more than 2^8 makes its warp rescale and redo
//               the first half before it is released.
// While softmax 1 works on S1(j) the tensor core computes O0 += P0 V_j and
// S0(j+1); while softmax 0 works on S0(j+1) it computes O1 += P1 V_j and
// S1(j+1).
//
// With a ticket counter the kernel is persistent: one CTA per SM takes work
// items (a whole unit, or one key range of a split unit) from the counter
// until none is left, the producer one item ahead, and hands each to the
// MMA and softmax warps through a two-slot ring in shared memory (a full
// and an empty mbarrier per slot).  Between items the K/V ring and the
// per-tile barriers run on; the producer reloads Q once the previous item's
// last S MMAs are done (B_QE).  The MMA warp reads the next item from the
// ring during the current item's last key tile and issues the next item's
// first S0 right after that tile's PV0 and its first S1 after PV1, as
// inside an item, so the two query tiles keep their alternation across
// items.  Each query tile's O is signalled complete on its own barrier
// (B_OF + i), and the next item's first P.V waits until both softmax
// warpgroups have read their O out (B_OE + i).
// Without a counter each CTA computes the one item blockIdx.x.
#pragma once

#include <type_traits>

#include "gemm_tc.cuh"

namespace mmh3 {

template <int HD>
struct Attn2Shape {
  static constexpr int kBoxBytes = 128 * 128;   // 128 rows x 128 bytes
  static constexpr int kHdBoxes = HD / 64;      // bf16 boxes across a head
  static constexpr int kTileBytes = kHdBoxes * kBoxBytes;
  static constexpr int kKV = 2;                 // K / V stages
  static constexpr int kQOff = 0;               // Q0 then Q1
  static constexpr int kKOff = 2 * kTileBytes;
  static constexpr int kVOff = kKOff + kKV * kTileBytes;
  static constexpr int kBarOff = kVOff + kKV * kTileBytes;
  static constexpr int kSmem = kBarOff + 512 + 1024;
  static constexpr int kThreads = 320;
  // floats per query row of a partial result: O[HD], m, l, padded to 16 bytes
  static constexpr int kPartStride = HD + 4;
  static constexpr size_t kPartBytesPerCta = (size_t)256 * kPartStride * 4;
};

// Eight partial maxima of a 128-score row (three-input max).
__device__ __forceinline__ void attn_row_max(const float (&s)[128], float (&pm)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) pm[i] = s[i];
#pragma unroll
  for (int k = 8; k < 120; k += 16)
#pragma unroll
    for (int i = 0; i < 8; ++i) pm[i] = fmax3(pm[i], s[k + i], s[k + 8 + i]);
#pragma unroll
  for (int i = 0; i < 8; ++i) pm[i] = fmaxf(pm[i], s[120 + i]);
}

__device__ __forceinline__ float attn_max8(const float (&pm)[8]) {
  return fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
}

// P = 2^(s * scale_log2 - m) for the keys of slices [H0, H1) (32 keys a
// slice) as bf16 pairs over the first 64 columns of S (16 columns a slice);
// the row sum accumulates in acc0 / acc1.  Scale/shift and the sum run as
// packed f32x2 operations; the exponentials stay on MUFU.  With kMaxHi (two
// slices), the maximum of the upper 64 scores (keys 64..127) is folded into
// pm alongside, one three-input maximum per pair of exponentials.
template <int H0, int H1, bool kMaxHi>
__device__ __forceinline__ void attn_exp_slices(const float (&s)[128], uint32_t ts, float scale_log2, float m,
                                                float2& acc0, float2& acc1, float (&pm)[8]) {
  static_assert(!kMaxHi || (H0 == 0 && H1 == 2), "the folded maximum runs alongside the lower half");
  const float2 sc2 = make_float2(scale_log2, scale_log2);
  const float2 nm2 = make_float2(-m, -m);
#pragma unroll
  for (int h = H0; h < H1; ++h) {
    uint32_t pk[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      if constexpr (kMaxHi) {
        const int g = h * 16 + q;
        pm[g & 7] = fmax3(pm[g & 7], s[64 + 2 * g], s[64 + 2 * g + 1]);
      }
      const int k = h * 32 + 2 * q;
      const float2 x = __ffma2_rn(make_float2(s[k], s[k + 1]), sc2, nm2);
      const float2 pv = make_float2(ex2_approx(x.x), ex2_approx(x.y));
      if (q & 1) acc1 = __fadd2_rn(acc1, pv);
      else acc0 = __fadd2_rn(acc0, pv);
      pk[q] = pack_bf16x2(pv.x, pv.y);
    }
    tmem_st16(ts + h * 16, pk);
  }
}

template <int HD>
__global__ void __launch_bounds__(320, 1)
    attn2_tc_kernel(const __grid_constant__ CUtensorMap tm, const __grid_constant__ CUtensorMap tmkv,
                    __nv_bfloat16* __restrict__ out, int ldo, int seq, int seq_kv, int k_off, int v_off,
                    float scale_log2, int heads, int whole, int split, int total, unsigned* __restrict__ ticket,
                    float* __restrict__ part, DevStatus* status, uint64_t limit_ns) {
  using Sh = Attn2Shape<HD>;
  constexpr int KV = Sh::kKV;
  constexpr uint32_t kIdescS = make_idesc(false, 128, 128, false, false);
  constexpr uint32_t kIdescO = make_idesc(false, 128, HD, false, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Sh::kBarOff);
  constexpr int B_Q = 0;
  constexpr int B_KF = 1, B_KE = B_KF + KV, B_VF = B_KE + KV, B_VE = B_VF + KV;
  constexpr int B_SF = B_VE + KV, B_PF = B_SF + 2, B_PH = B_PF + 2, B_OF = B_PH + 2, B_DRAIN = B_OF + 2;
  constexpr int B_QE = B_DRAIN + 1, B_OE = B_QE + 1, B_IF = B_OE + 2, B_IE = B_IF + 2;
  constexpr int kNumBars = B_IE + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* items = reinterpret_cast<volatile int*>(tmem_slot + 2);  // the two-slot work ring

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = smem_u32(bars);
  auto bar = [&](int i) { return bar0 + 8u * i; };

  // Queries: rows [z*seq, (z+1)*seq) of the panel `tm` (q at column 0).
  // Keys / values: rows [z*seq_kv, (z+1)*seq_kv) of `tmkv`, k at column
  // k_off, v at v_off (the same panel for a whole sequence on one GPU; the
  // gathered K|V rows of all ranks for a sequence split over ranks).
  // Work item w < total.  Items [0, whole) are whole units u = w (256
  // query rows of one head of one sequence, u = (zseq*heads + head)*nq +
  // qpair, all key tiles).  The rest are the tail: item whole + b, b = t *
  // split + piece, computes key range `piece` of the `split` contiguous
  // ranges of unit whole + t and writes its unnormalised partial result to
  // part slot b for attn_merge_kernel.
  const int nq = (seq + 255) / 256;
  const int kv_tiles = (seq_kv + 127) / 128;
  struct Item {
    int u, j0, n, tb;  // unit, first key tile, key tiles, tail index (< 0: whole)
  };
  auto item_of = [&](int w) {
    Item it;
    it.tb = w - whole;
    const int sp = it.tb < 0 ? 1 : split;
    it.u = it.tb < 0 ? w : whole + it.tb / split;
    const int piece = it.tb < 0 ? 0 : it.tb % split;
    it.j0 = piece * kv_tiles / sp;
    it.n = (piece + 1) * kv_tiles / sp - it.j0;
    return it;
  };
  struct Unit {
    int head, qpair, seq_row0, kv_row0, q_row0;
  };
  auto unit_of = [&](int u) {
    Unit r;
    r.qpair = u % nq;
    r.head = (u / nq) % heads;
    const int zseq = u / (nq * heads);
    r.seq_row0 = zseq * seq;
    r.kv_row0 = zseq * seq_kv;
    r.q_row0 = r.seq_row0 + r.qpair * 256;
    return r;
  };

  if (threadIdx.x == 0) {
    mbar_init(bar(B_Q), 1);
    for (int s = 0; s < KV; ++s) {
      mbar_init(bar(B_KF + s), 1);
      mbar_init(bar(B_KE + s), 1);
      mbar_init(bar(B_VF + s), 1);
      mbar_init(bar(B_VE + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_SF + i), 1);
      mbar_init(bar(B_PF + i), 128);
      mbar_init(bar(B_PH + i), 128);
      mbar_init(bar(B_IF + i), 1);
      mbar_init(bar(B_IE + i), 9);  // the MMA warp and the eight softmax warps
      mbar_init(bar(B_OF + i), 1);
      mbar_init(bar(B_OE + i), 128);
    }
    mbar_init(bar(B_DRAIN), 1);
    mbar_init(bar(B_QE), 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch(&tm);
    tma_prefetch(&tmkv);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 512);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait();
  // S_i at columns 128 i, O_i at 256 + HD i
  auto t_s = [&](int i) { return tmem + 128u * i; };
  auto t_o = [&](int i) { return tmem + 256u + (uint32_t)HD * i; };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      // Takes the CTA's items from the ticket counter (one ahead, so the
      // atomic's latency hides behind the current item) and hands each to
      // the other roles through the work ring.  Per item: Q0 and Q1 (once
      // the previous item's S MMAs have read the old ones), then its K / V
      // tiles through the two-stage ring, whose counter c runs on across
      // items.  Without a counter the CTA's one item is blockIdx.x.
      const bool chk = status != nullptr && status->check != 0;
      int c = 0, in_k = 0, in_v = 0, q_last = -1;
      bool q_pending = false;  // a Q copy no role has waited for yet (the last one)
      bool ok = true;
      unsigned next = ticket != nullptr ? atomicAdd(ticket, 1u) : blockIdx.x;
      for (int k = 0; ok; ++k) {
        const int w = next < (unsigned)total ? (int)next : total;
        // slot k & 1 is free once every role has read item k - 2
        if (!mbar_wait_ab(bar(B_IE + (k & 1)), (uint32_t)(((k >> 1) & 1) ^ 1), limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        items[k & 1] = w;
        mbar_arrive(bar(B_IF + (k & 1)));
        if (w >= total) break;
        next = ticket != nullptr ? atomicAdd(ticket, 1u) : (unsigned)total;
        const Item it = item_of(w);
        const Unit un = unit_of(it.u);
        const int xq = un.head * HD, xk = k_off + un.head * HD, xv = v_off + un.head * HD;
        // MMH3_CHECK mode: the x coordinates of every copy of the item and
        // the first rows of Q and of its keys (the key rows only grow from
        // there); a failure issues nothing
        if (chk) {
          bool fine = true;
          for (int cc = 0; cc < Sh::kHdBoxes && fine; ++cc)
            fine = tma_coords_ok(status, true, xq + cc * 64, un.q_row0, 2) &&
                   tma_coords_ok(status, true, xk + cc * 64, un.kv_row0 + it.j0 * 128, 2) &&
                   tma_coords_ok(status, true, xv + cc * 64, un.kv_row0 + it.j0 * 128, 2);
          if (!fine) {
            *abort_flag = 1;
            ok = false;
            break;
          }
        }
        if (k > 0 && !mbar_wait_ab(bar(B_QE), (uint32_t)((k - 1) & 1), limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        mbar_expect_tx(bar(B_Q), 2 * Sh::kTileBytes);
        for (int i = 0; i < 2; ++i)
          for (int cc = 0; cc < Sh::kHdBoxes; ++cc)
            tma_load_2d(sbase + Sh::kQOff + i * Sh::kTileBytes + cc * Sh::kBoxBytes, &tm, bar(B_Q),
                        xq + cc * 64, un.q_row0 + 128 * i);
        q_last = k;
        q_pending = true;
        for (int j = it.j0; j < it.j0 + it.n && ok; ++j, ++c) {
          const int s = c % KV;
          const uint32_t ph = (uint32_t)((c / KV) & 1);
          const int y = un.kv_row0 + j * 128;
          if (!mbar_wait_ab(bar(B_KE + s), ph ^ 1u, limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          mbar_expect_tx(bar(B_KF + s), Sh::kTileBytes);
          for (int cc = 0; cc < Sh::kHdBoxes; ++cc)
            tma_load_2d(sbase + Sh::kKOff + s * Sh::kTileBytes + cc * Sh::kBoxBytes, &tmkv, bar(B_KF + s),
                        xk + cc * 64, y);
          in_k = c + 1;
          if (!mbar_wait_ab(bar(B_VE + s), ph ^ 1u, limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          mbar_expect_tx(bar(B_VF + s), Sh::kTileBytes);
          for (int cc = 0; cc < Sh::kHdBoxes; ++cc)
            tma_load_2d(sbase + Sh::kVOff + s * Sh::kTileBytes + cc * Sh::kBoxBytes, &tmkv, bar(B_VF + s),
                        xv + cc * 64, y);
          in_v = c + 1;
        }
      }
      if (!ok) {
        if (!*abort_flag) record_error(status, DEV_TIMEOUT_PRODUCER, c);
        *abort_flag = 1;
        // let the copies still in flight land (bounded) before the CTA's
        // shared memory is released
        if (q_pending) mbar_wait(bar(B_Q), (uint32_t)(q_last & 1), limit_ns);
        for (int i = (in_k > KV ? in_k - KV : 0); i < in_k; ++i)
          mbar_wait(bar(B_KF + i % KV), (uint32_t)((i / KV) & 1), limit_ns);
        for (int i = (in_v > KV ? in_v - KV : 0); i < in_v; ++i)
          mbar_wait(bar(B_VF + i % KV), (uint32_t)((i / KV) & 1), limit_ns);
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------- MMA issuer
    // The whole warp runs this loop and its waits, so descriptors and
    // tensor-memory addresses are warp-uniform; one elected lane (always the
    // same) issues every MMA and commit.  Stage indices are compile-time
    // (the loop body is instantiated per K/V stage), so each descriptor is a
    // base plus a constant.
    // Order within an item: S0(0) S1(0) | PV0(0) S0(1) PV1(0) S1(1) |
    // PV0(1) S0(2) ...  S_i(j+1) goes right after PV_i(j), so the tensor
    // core computes S0(j+1) while softmax 1 still works on S1(j).  Each
    // PV_i(j) is issued in two halves of 64 keys, the first once P_i's first
    // half is released.  The key-tile counter c (stages and barrier phases)
    // runs on across items; an item's first S MMAs follow the previous
    // item's last P.V, so they overlap that item's epilogue.
    static_assert(KV == 2, "the issue loop is written for two K/V stages");
    const uint64_t dk_major = sdesc_sw128(sbase, 16, 1024);           // Q, K: K-major
    const uint64_t dv_major = sdesc_sw128(sbase, Sh::kBoxBytes, 1024);  // V: MN-major
    auto wait = [&](int b, uint32_t ph) {
      return __all_sync(0xffffffffu, mbar_wait_ab(bar(b), ph, limit_ns, abort_flag));
    };
    auto issue_s = [&](int i, auto stage) {
      constexpr int st = decltype(stage)::value;
#pragma unroll
      for (int ks = 0; ks < HD / 16; ++ks) {
        const uint32_t off = (ks / 4) * Sh::kBoxBytes + (ks % 4) * 32;
        umma_ss_elect(t_s(i), dk_major + ((Sh::kQOff + i * Sh::kTileBytes + off) >> 4),
                      dk_major + ((Sh::kKOff + st * Sh::kTileBytes + off) >> 4), kIdescS, ks > 0 ? 1u : 0u);
      }
      umma_commit_elect(bar(B_SF + i));
    };
    auto issue_pv = [&](int i, int half, bool first, auto stage) {
      constexpr int st = decltype(stage)::value;
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        const int ks = half * 4 + k4;
        umma_ts_elect(t_o(i), t_s(i) + ks * 8, dv_major + ((Sh::kVOff + st * Sh::kTileBytes + ks * 16 * 128) >> 4),
                      kIdescO, (!first || ks > 0) ? 1u : 0u);
      }
    };
    // Key tile j of an item of n tiles (item k), counter c, in stage st:
    // PV0(j) [S0(j+1)] PV1(j) [S1(j+1)].  The item's first P.V overwrites O,
    // so it waits until the softmax warps have read the previous item's O.
    auto step = [&](int k, int j, int n, int c, auto stage) -> bool {
      constexpr int st = decltype(stage)::value;
      const std::integral_constant<int, 1 - st> next{};
      const uint32_t pj = (uint32_t)(c & 1);
      const uint32_t pv = (uint32_t)((c / KV) & 1);
      const bool more = j + 1 < n;
      if (j == 0 && k > 0 && (!wait(B_OE + 0, (uint32_t)((k - 1) & 1)) || !wait(B_OE + 1, (uint32_t)((k - 1) & 1))))
        return false;
      if (!wait(B_VF + st, pv) || !wait(B_PH + 0, pj)) return false;
      tc_fence_after();
      issue_pv(0, 0, j == 0, stage);
      if (!wait(B_PF + 0, pj)) return false;
      tc_fence_after();
      issue_pv(0, 1, j == 0, stage);
      if (more) {
        if (!wait(B_KF + 1 - st, (uint32_t)(((c + 1) / KV) & 1))) return false;
        tc_fence_after();
        issue_s(0, next);
      }
      if (!wait(B_PH + 1, pj)) return false;
      tc_fence_after();
      issue_pv(1, 0, j == 0, stage);
      if (!wait(B_PF + 1, pj)) return false;
      tc_fence_after();
      issue_pv(1, 1, j == 0, stage);
      umma_commit_elect(bar(B_VE + st));
      if (more) {
        issue_s(1, next);
        umma_commit_elect(bar(B_KE + 1 - st));
        // the item's last S MMAs: once they are done, the producer may load
        // the next item's Q while this tile's softmax and P.V run
        if (j + 2 == n) umma_commit_elect(bar(B_QE));
      }
      return true;
    };
    // The item's last key tile (j = n - 1): PV0 and PV1 as in step, each
    // query tile's O signalled complete on its own barrier (B_OF + i) right
    // after its last P.V, and, when a next item follows (n_next > 0 key
    // tiles), that item's first S0 issued right after PV0 and its first S1
    // after PV1, as inside an item, so the two query tiles keep their
    // alternation across items.
    auto last_step = [&](int k, int j, int c, int n_next, auto stage) -> bool {
      constexpr int st = decltype(stage)::value;
      const std::integral_constant<int, 1 - st> next{};
      const uint32_t pj = (uint32_t)(c & 1);
      const uint32_t pv = (uint32_t)((c / KV) & 1);
      if (j == 0 && k > 0 && (!wait(B_OE + 0, (uint32_t)((k - 1) & 1)) || !wait(B_OE + 1, (uint32_t)((k - 1) & 1))))
        return false;
      if (!wait(B_VF + st, pv) || !wait(B_PH + 0, pj)) return false;
      tc_fence_after();
      issue_pv(0, 0, j == 0, stage);
      if (!wait(B_PF + 0, pj)) return false;
      tc_fence_after();
      issue_pv(0, 1, j == 0, stage);
      umma_commit_elect(bar(B_OF + 0));
      if (n_next > 0) {
        if (!wait(B_Q, (uint32_t)((k + 1) & 1)) || !wait(B_KF + 1 - st, (uint32_t)(((c + 1) / KV) & 1))) return false;
        tc_fence_after();
        issue_s(0, next);
      }
      if (!wait(B_PH + 1, pj)) return false;
      tc_fence_after();
      issue_pv(1, 0, j == 0, stage);
      if (!wait(B_PF + 1, pj)) return false;
      tc_fence_after();
      issue_pv(1, 1, j == 0, stage);
      umma_commit_elect(bar(B_VE + st));
      umma_commit_elect(bar(B_OF + 1));
      if (n_next > 0) {
        issue_s(1, next);
        umma_commit_elect(bar(B_KE + 1 - st));
        if (n_next == 1) umma_commit_elect(bar(B_QE));  // the next item's only S MMAs
      }
      return true;
    };
    const std::integral_constant<int, 0> stage0{};
    const std::integral_constant<int, 1> stage1{};
    // item kk from the work ring (warp-uniform); false on timeout
    auto fetch = [&](int kk, int& w_out) -> bool {
      if (!wait(B_IF + (kk & 1), (uint32_t)((kk >> 1) & 1))) return false;
      w_out = items[kk & 1];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_IE + (kk & 1)));
      return true;
    };
    int c = 0;
    int w = total;
    bool ok = fetch(0, w);
    bool s_issued = false;  // the item's first S MMAs went out with the previous item's last tile
    for (int k = 0; ok && w < total; ++k) {
      const int n = item_of(w).n;
      if (!s_issued) {
        if (!wait(B_Q, (uint32_t)(k & 1)) || !wait(B_KF + (c & 1), (uint32_t)((c / KV) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (c & 1) {
          issue_s(0, stage1);
          issue_s(1, stage1);
        } else {
          issue_s(0, stage0);
          issue_s(1, stage0);
        }
        umma_commit_elect(bar(B_KE + (c & 1)));
        if (n == 1) umma_commit_elect(bar(B_QE));  // no further S MMA reads this Q
      }
      for (int j = 0; j + 1 < n && ok; ++j, ++c) ok = (c & 1) ? step(k, j, n, c, stage1) : step(k, j, n, c, stage0);
      if (!ok) break;
      int w_next = total;
      if (!fetch(k + 1, w_next)) {
        ok = false;
        break;
      }
      const int n_next = w_next < total ? item_of(w_next).n : 0;
      ok = (c & 1) ? last_step(k, n - 1, c, n_next, stage1) : last_step(k, n - 1, c, n_next, stage0);
      ++c;
      s_issued = n_next > 0;
      w = w_next;
    }
    if (!ok) {
      if (lane == 0 && !*abort_flag) record_error(status, DEV_TIMEOUT_MMA, blockIdx.x);
      __syncwarp();
      *abort_flag = 1;
      umma_commit_elect(bar(B_DRAIN));
      mbar_wait(bar(B_DRAIN), 0, limit_ns);
    }
  } else {
    // -------------------------------------------------- softmax warpgroups
    const int wg = (warp - 2) >> 2;       // query tile
    const int lgrp = warp & 3;            // TMEM lane quarter
    const int r = lgrp * 32 + lane;       // row within the tile
    const uint32_t lane_off = (uint32_t)(lgrp * 32) << 16;
    const uint32_t ts = t_s(wg) + lane_off;
    const uint32_t to = t_o(wg) + lane_off;
    int c = 0;
    // item k = w: its key tiles are c .. c_end - 1 of the CTA's count;
    // valid = keys of its first tile that exist
    auto body = [&](int k, int w, int valid, int c_end) -> bool {
      float m_ref = 0.f, l_sum = 0.f;
      for (bool first = true; c < c_end; ++c, valid -= 128, first = false) {
        {
          const bool fail = !mbar_wait_ab(bar(B_SF + wg), (uint32_t)(c & 1), limit_ns, abort_flag);
          if (__any_sync(0xffffffffu, fail)) return false;
        }
        tc_fence_after();
        float s[128];
        {
          uint32_t u0[32], u1[32], u2[32], u3[32];
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
        if (valid < 128) {
#pragma unroll
          for (int kk = 0; kk < 128; ++kk)
            if (kk >= valid) s[kk] = -INFINITY;
        }
        float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
        float pm[8];
        if (first) {
          // first key tile: the row maximum before any exponential
          attn_row_max(s, pm);
          m_ref = attn_max8(pm) * scale_log2;
          attn_exp_slices<0, 2, false>(s, ts, scale_log2, m_ref, acc0, acc1, pm);
        } else {
          // keys 0..63 against the current reference, with the maximum of
          // keys 64..127 folded in.  The lower half needs no maximum of its
          // own: its exponentials are non-negative, so a lower-half sum of at
          // most 2^8 bounds each of them by 2^8, i.e. no lower score exceeds
          // the reference by more than 8 (log2 domain).  A row whose lower
          // sum or upper maximum fails that bound rescales to its full row
          // maximum and redoes the lower half.
#pragma unroll
          for (int i = 0; i < 8; ++i) pm[i] = -INFINITY;
          attn_exp_slices<0, 2, true>(s, ts, scale_log2, m_ref, acc0, acc1, pm);
          const float m_hi = attn_max8(pm) * scale_log2;
          const float lo_sum = (acc0.x + acc0.y) + (acc1.x + acc1.y);
          const bool need = lo_sum > 256.0f || m_hi > m_ref + 8.0f;
          if (__any_sync(0xffffffffu, need)) {
            // O_i holds every earlier product of the item (see the kernel comment).
            attn_row_max(s, pm);
            const float m_new = need ? fmaxf(attn_max8(pm) * scale_log2, m_ref) : m_ref;
            const float f = ex2_approx(m_ref - m_new);
            l_sum *= f;
            m_ref = m_new;
#pragma unroll 1
            for (int cc = 0; cc < HD / 16; ++cc) {
              uint32_t uu[16];
              tmem_ld16(to + cc * 16, uu);
              tmem_wait_ld();
#pragma unroll
              for (int i2 = 0; i2 < 16; ++i2) uu[i2] = __float_as_uint(__uint_as_float(uu[i2]) * f);
              tmem_st16(to + cc * 16, uu);
            }
            tmem_wait_st();
            acc0 = make_float2(0.f, 0.f);
            acc1 = make_float2(0.f, 0.f);
            attn_exp_slices<0, 2, false>(s, ts, scale_log2, m_ref, acc0, acc1, pm);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(B_PH + wg));
        attn_exp_slices<2, 4, false>(s, ts, scale_log2, m_ref, acc0, acc1, pm);
        l_sum += (acc0.x + acc0.y) + (acc1.x + acc1.y);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(B_PF + wg));
      }
      {
        const bool fail = !mbar_wait_ab(bar(B_OF + wg), (uint32_t)(k & 1), limit_ns, abort_flag);
        if (__any_sync(0xffffffffu, fail)) return false;
      }
      tc_fence_after();
      const Item it = item_of(w);
      const Unit un = unit_of(it.u);
      const int qr = un.qpair * 256 + wg * 128 + r;
      const bool row_ok = qr < seq;
      if (it.tb < 0) {
        const float inv = l_sum > 0.f ? 1.0f / l_sum : 0.f;
        __nv_bfloat16* dst = out + (size_t)(un.seq_row0 + qr) * ldo + un.head * HD;
#pragma unroll 1
        for (int cc = 0; cc < HD / 32; ++cc) {
          float v[32];
          ld_acc32(to + cc * 32, v);
#pragma unroll
          for (int i2 = 0; i2 < 32; ++i2) v[i2] *= inv;
          if (row_ok) store32(dst + cc * 32, v);
        }
      } else {
        // partial: O unnormalised (relative to m_ref), then m_ref and l_sum
        float* dst = part + ((size_t)it.tb * 256 + wg * 128 + r) * Sh::kPartStride;
#pragma unroll 1
        for (int cc = 0; cc < HD / 32; ++cc) {
          float v[32];
          ld_acc32(to + cc * 32, v);
          if (row_ok) store32(dst + cc * 32, v);
        }
        if (row_ok) {
          dst[HD] = m_ref;
          dst[HD + 1] = l_sum;
        }
      }
      // this thread's O is read: the next item's first P.V may overwrite it
      tc_fence_before();
      mbar_arrive(bar(B_OE + wg));
      return true;
    };
    bool ok = true;
    for (int k = 0; ok; ++k) {
      {
        const bool fail = !mbar_wait_ab(bar(B_IF + (k & 1)), (uint32_t)((k >> 1) & 1), limit_ns, abort_flag);
        if (__any_sync(0xffffffffu, fail)) {
          ok = false;
          break;
        }
      }
      const int w = items[k & 1];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_IE + (k & 1)));
      if (w >= total) break;
      const Item it = item_of(w);
      ok = body(k, w, seq_kv - it.j0 * 128, c + it.n);
    }
    if (!ok) {
      if (lane == 0 && !*abort_flag) record_error(status, DEV_TIMEOUT_SOFTMAX, blockIdx.x);
      *abort_flag = 1;
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Combine the `split` partial results of each tail unit (unnormalised O,
// reference maximum m in the log2 domain, row sum l):
//   m* = max_p m_p,  w_p = 2^(m_p - m*),  O = sum_p w_p O_p / sum_p w_p l_p.
// One warp per query row (each lane four of the head's columns, so a warp
// reads a partial row as whole lines); a CTA of 8 warps covers 8 rows of a
// unit, 32 CTAs a unit.
template <int HD>
__global__ void __launch_bounds__(256) attn_merge_kernel(const float* __restrict__ part, int split,
                                                         __nv_bfloat16* __restrict__ out, int ldo, int seq,
                                                         int heads, int unit0) {
  pdl_launch_dependents();
  pdl_wait();
  static_assert(HD == 128 || HD == 64, "head_dim");
  constexpr int kLaneCols = HD / 32;  // 4 or 2
  const int nq = (seq + 255) / 256;
  const int t = blockIdx.x / 32;
  const int u = unit0 + t;
  const int qpair = u % nq;
  const int head = (u / nq) % heads;
  const int zseq = u / (nq * heads);
  const int r = (blockIdx.x % 32) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int qr = qpair * 256 + r;
  if (qr >= seq) return;
  auto row = [&](int p) {
    return part + ((size_t)(t * split + p) * 256 + r) * Attn2Shape<HD>::kPartStride;
  };
  float m = -INFINITY;
  for (int p = 0; p < split; ++p) m = fmaxf(m, row(p)[HD]);
  float l = 0.f;
  float acc[kLaneCols];
#pragma unroll
  for (int i = 0; i < kLaneCols; ++i) acc[i] = 0.f;
  for (int p = 0; p < split; ++p) {
    const float* rp = row(p);
    const float wgt = ex2_approx(rp[HD] - m);
    l = fmaf(wgt, rp[HD + 1], l);
#pragma unroll
    for (int i = 0; i < kLaneCols; ++i) acc[i] = fmaf(wgt, rp[lane * kLaneCols + i], acc[i]);
  }
  const float inv = l > 0.f ? 1.0f / l : 0.f;
  __nv_bfloat16* dst = out + (size_t)(zseq * seq + qr) * ldo + head * HD + lane * kLaneCols;
  if constexpr (kLaneCols == 4) {
    uint2 v;
    v.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    v.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2*>(dst) = v;
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  }
}

}  // namespace mmh3
