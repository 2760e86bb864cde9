// The C ABI entry points that run the hot path: adaLN modulation, the
// modulated block, the 50-block stack with its output heads, the SigLIP
// encoder layer, and around them the token refiner, the embed and output
// unpacking, one whole denoise evaluation, the block over a sequence shard
// and the block on host buffers.  Each entry point validates everything
// before the first launch and then enqueues a fixed sequence of kernels on
// the caller's stream(s) (no host synchronisation, no allocation).
//
// Step order follows "cortiq_engine/mmh3.rs" (cortiq-engine 0.5.72):
// MiniMaxH3::forward ("embed", "blocks", "heads"), refine_text,
// block_forward and ffn_tail;
// the encoder layer follows "ffai-argus 0.7.0 src/siglip.rs",
// Layer::forward and finish_attention.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "mmh3_internal.h"

using namespace mmh3;


// --------------------------------------------------------------- profiler
// Per-phase device time of the block, in the nine slots of the reference's
// phase profile ("cortiq_engine/mmh3.rs", MMH3_PROF): 0 norm+modulate (with
// the adaLN curve and the rotation table), 1 qkv GEMM (qk-norm and rotation
// are fused into it, so slot 2 stays 0), 3 attention, 4 out GEMM with the
// gated residual, 5 fc1 GEMM with SwiGLU (slot 6 stays 0), 7 fc2 GEMM with
// the gated residual (slot 8 stays 0).  Enabled by mmh3_prof_enable(1);
// events are recorded on the caller's stream between the launches, so the
// phases never overlap and are never counted twice.
// Each interval also carries the kernel it times (MMH3_PROF_K_*), so the
// memory-bound kernels that share slot 0 get their own device times.
struct ProfRec {
  int slot;
  int kernel;
  cudaEvent_t a, b;
};
static bool g_prof_on = false;
static std::vector<ProfRec> g_prof_recs;
static std::vector<cudaEvent_t> g_prof_free;
static double g_prof_ms[9] = {0};
static double g_prof_kms[MMH3_PROF_KERNELS] = {0};
static long g_prof_kcalls[MMH3_PROF_KERNELS] = {0};
static long g_prof_blocks = 0;

static cudaEvent_t prof_event() {
  cudaEvent_t e = nullptr;
  if (!g_prof_free.empty()) {
    e = g_prof_free.back();
    g_prof_free.pop_back();
  } else if (cudaEventCreate(&e) != cudaSuccess) {
    e = nullptr;
  }
  return e;
}

struct PhaseMark {
  cudaEvent_t last = nullptr;
  cudaStream_t s;
  bool on;
  PhaseMark(cudaStream_t st, bool enabled) : s(st), on(enabled && g_prof_on) {
    if (on && (last = prof_event()) != nullptr) cudaEventRecord(last, s);
  }
  // closes the running interval as phase `slot`, kernel `kernel`, and opens
  // the next one
  void mark(int slot, int kernel) {
    if (!on || last == nullptr) return;
    cudaEvent_t e = prof_event();
    if (e == nullptr) return;
    cudaEventRecord(e, s);
    g_prof_recs.push_back({slot, kernel, last, e});
    cudaEvent_t next = prof_event();
    if (next) cudaEventRecord(next, s);
    last = next;
  }
  ~PhaseMark() {
    if (last) g_prof_free.push_back(last);
  }
};

namespace {

struct Workspace {
  float* mods;
  float2* cs;
  void* xn1;
  void* qkv;
  void* attn;
  void* xn2;
  void* act;
  void* head;
  float* fmods;
  unsigned* sched;  // attention's work counter (zeroed by the block's first RMSNorm)
  size_t bytes;
  CanaryList canaries;  // MMH3_CHECK mode: one after each region
};

Workspace carve(const mmh3_dims& d, int n, void* base) {
  const size_t es = (size_t)esize_of(d.act_dtype);
  const size_t H = (size_t)d.hidden, I = (size_t)d.heads * d.head_dim, F = (size_t)d.ffn;
  const size_t N = (size_t)n;
  Workspace w{};
  size_t off = 0;
  const bool canary = check_mode();
  auto take = [&](size_t bytes) {
    uint8_t* p = static_cast<uint8_t*>(base) + off;
    off += align256(bytes);
    if (canary) {
      if (base && w.canaries.n < kMaxCanaries)
        w.canaries.p[w.canaries.n++] = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(base) + off);
      off += kCanaryBytes;
    }
    return base ? static_cast<void*>(p) : nullptr;
  };
  w.mods = static_cast<float*>(take(2 * 3 * 6 * H * 4));
  w.cs = static_cast<float2*>(take(N * 3 * (size_t)d.rope_k * 8));
  w.xn1 = take(N * H * es);
  w.qkv = take(N * 3 * I * es);
  w.attn = take(N * I * es);
  w.xn2 = take(N * H * es);
  w.act = take(N * F * es);
  w.head = take(N * H * es);
  w.fmods = static_cast<float*>(take(2 * 2 * H * 4));
  w.sched = static_cast<unsigned*>(take(16));
  w.bytes = off;
  return w;
}

bool misaligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) != 0; }

mmh3_status check_dims(const mmh3_dims* d) {
  if (d == nullptr) return fail(MMH3_ERR_ARG, "dims is null");
  if (d->act_dtype != MMH3_BF16 && d->act_dtype != MMH3_F32) return fail(MMH3_ERR_ARG, "act_dtype %d", d->act_dtype);
  if (d->hidden <= 0 || d->hidden % 128 != 0 || d->hidden > 4096)
    return fail(MMH3_ERR_SHAPE, "hidden %d must be a positive multiple of 128 (<= 4096)", d->hidden);
  if (d->head_dim != 64 && d->head_dim != 128) return fail(MMH3_ERR_SHAPE, "head_dim %d not in {64, 128}", d->head_dim);
  if (d->act_dtype == MMH3_F32 && d->head_dim != 64)
    return fail(MMH3_ERR_UNSUPPORTED, "fp32 activations support head_dim 64 only");
  if (d->heads <= 0 || d->heads > 256)
    return fail(MMH3_ERR_SHAPE, "heads = %d not in [1, 256]", d->heads);
  if (d->ffn <= 0 || d->ffn % 128 != 0) return fail(MMH3_ERR_SHAPE, "ffn %d must be a multiple of 128", d->ffn);
  if (d->rank < 1 || d->rank > 32) return fail(MMH3_ERR_SHAPE, "rank %d not in [1, 32]", d->rank);
  if (d->grid < 2) return fail(MMH3_ERR_SHAPE, "grid %d < 2", d->grid);
  if (d->rope_k != d->head_dim / 8) return fail(MMH3_ERR_SHAPE, "rope_k %d != head_dim/8", d->rope_k);
  if (!(d->eps > 0) || !(d->qk_eps > 0)) return fail(MMH3_ERR_ARG, "eps must be positive");
  return MMH3_OK;
}

mmh3_status check_block(const mmh3_dims& d, const mmh3_block_weights* w, bool modulated) {
  if (w == nullptr) return fail(MMH3_ERR_ARG, "block weights are null");
  const void* req[] = {w->norm1, w->norm2, w->wqkv, w->wout, w->q_norm, w->k_norm, w->wfc1, w->wfc2};
  for (const void* p : req) {
    if (p == nullptr) return fail(MMH3_ERR_ARG, "a block weight pointer is null");
    if (misaligned(p)) return fail(MMH3_ERR_ALIGN, "a block weight pointer is not 16-byte aligned");
  }
  if (modulated) {
    const void* ad[] = {w->adaln_w, w->adaln_b, w->adaln_table};
    for (const void* p : ad) {
      if (p == nullptr) return fail(MMH3_ERR_ARG, "adaLN pointer is null in a modulated block");
      if (misaligned(p)) return fail(MMH3_ERR_ALIGN, "adaLN pointer is not 16-byte aligned");
    }
  }
  (void)d;
  return MMH3_OK;
}

// MMH3_CHECK mode: fill the workspace canaries (verify = false) or check
// them after the kernel kid (verify = true); nothing without canaries.
mmh3_status canaries(const Workspace& ws, bool verify, int kid, cudaStream_t s) {
  if (ws.canaries.n == 0) return MMH3_OK;
  cudaError_t e = launch_canary(ws.canaries, verify, kid, s);
  return e == cudaSuccess ? MMH3_OK : cuda_fail(e, "canary launch");
}

// norm1-modulate -> qkv+qknorm+rope (the part before attention)
mmh3_status block_pre(const mmh3_dims& d, const mmh3_block_weights& w, const float* x, int n, const Plan& plan,
                      const float* mods, const float2* cs, const Workspace& ws, cudaStream_t s, PhaseMark& pm) {
  const int H = d.hidden, I = d.heads * d.head_dim;
  const int dt = d.act_dtype;
  const int stride = 6 * H;
  cudaError_t e = launch_norm_mod(dt, x, n, H, w.norm1, d.eps, mods, stride, 0 * H, 1 * H, plan.block_rows, 0,
                                  ws.xn1, s, ws.sched);
  if (e != cudaSuccess) return cuda_fail(e, "norm1/modulate launch");
  pm.mark(0, MMH3_PROF_K_NORM1);
  mmh3_status st = canaries(ws, true, MMH3_PROF_K_NORM1, s);
  if (st != MMH3_OK) return st;
  st = gemm_qkv(dt, ws.xn1, w.wqkv, n, 3 * I, H, d.head_dim, I, w.q_norm, w.k_norm, cs, d.qk_eps, ws.qkv, s);
  if (st != MMH3_OK) return st;
  pm.mark(1, MMH3_PROF_K_QKV);
  return canaries(ws, true, MMH3_PROF_K_QKV, s);
}

// attention -> out+gated residual -> norm2-modulate -> fc1+SwiGLU -> fc2+gated
// residual.  kv_all == nullptr: keys and values from this call's own qkv
// panel; otherwise from kv_all [n_kv, 2*inner] (the gathered K|V rows).
mmh3_status block_post(const mmh3_dims& d, const mmh3_block_weights& w, float* x, int n, const Plan& plan,
                       const float* mods, const Workspace& ws, cudaStream_t s, PhaseMark& pm,
                       const void* kv_all, int n_kv) {
  const int H = d.hidden, I = d.heads * d.head_dim, F = d.ffn;
  const int dt = d.act_dtype;
  const int stride = 6 * H;
  const float scale = 1.0f / std::sqrt((float)d.head_dim);
  // the SwiGLU activation region is free until fc1: it holds the partial
  // results of split attention units
  const size_t act_bytes = (size_t)n * F * esize_of(dt);
  mmh3_status st = kv_all == nullptr
                       ? attention(dt, ws.qkv, 1, n, d.heads, d.head_dim, scale, ws.attn, s, ws.act, act_bytes,
                                   ws.sched)
                       : attention_kv(dt, ws.qkv, n, kv_all, n_kv, d.heads, d.head_dim, scale, ws.attn, s, ws.act,
                                      act_bytes, ws.sched);
  if (st != MMH3_OK) return st;
  pm.mark(3, MMH3_PROF_K_ATTN);
  st = canaries(ws, true, MMH3_PROF_K_ATTN, s);
  if (st != MMH3_OK) return st;
  st = gemm_gated_residual(dt, ws.attn, w.wout, n, H, I, x, mods, stride, 2 * H, plan.block_rows, s);
  if (st != MMH3_OK) return st;
  pm.mark(4, MMH3_PROF_K_OUT);
  st = canaries(ws, true, MMH3_PROF_K_OUT, s);
  if (st != MMH3_OK) return st;
  cudaError_t e = launch_norm_mod(dt, x, n, H, w.norm2, d.eps, mods, stride, 3 * H, 4 * H, plan.block_rows, 0,
                                  ws.xn2, s);
  if (e != cudaSuccess) return cuda_fail(e, "norm2/modulate launch");
  pm.mark(0, MMH3_PROF_K_NORM2);
  st = canaries(ws, true, MMH3_PROF_K_NORM2, s);
  if (st != MMH3_OK) return st;
  st = gemm_swiglu(dt, ws.xn2, w.wfc1, n, F, H, ws.act, s);
  if (st != MMH3_OK) return st;
  pm.mark(5, MMH3_PROF_K_FC1);
  st = canaries(ws, true, MMH3_PROF_K_FC1, s);
  if (st != MMH3_OK) return st;
  st = gemm_gated_residual(dt, ws.act, w.wfc2, n, H, F, x, mods, stride, 5 * H, plan.block_rows, s);
  if (st != MMH3_OK) return st;
  pm.mark(7, MMH3_PROF_K_FC2);
  if (pm.on) ++g_prof_blocks;
  return canaries(ws, true, MMH3_PROF_K_FC2, s);
}

// The whole block on one GPU.
mmh3_status block_core(const mmh3_dims& d, const mmh3_block_weights& w, float* x, int n,
                       const Plan& plan, const float* mods, const float2* cs, const Workspace& ws,
                       cudaStream_t s, PhaseMark& pm) {
  mmh3_status st = block_pre(d, w, x, n, plan, mods, cs, ws, s, pm);
  if (st != MMH3_OK) return st;
  return block_post(d, w, x, n, plan, mods, ws, s, pm, nullptr, 0);
}

// The block's own adaLN basis has two timestep slots (rows [slot][tag]
// [chunk][H], slot s at ts[s]); how a third or fourth distinct timestep
// (keyframe or reference rows on their condition clocks) maps onto it is
// not fixed, so such plans run only with a caller's modulation.
mmh3_status own_curve_slots(const Plan& plan) {
  if (plan.n_ts > 2)
    return fail(MMH3_ERR_UNSUPPORTED,
                "%d distinct timesteps: the adaLN basis holds two slots; pass the modulation (mods_or_null)",
                plan.n_ts);
  return MMH3_OK;
}

// adaLN modulation of one block (when own_mods) into ws.mods and the
// rotation table (when pos != null) into ws.cs, in one launch.
mmh3_status prologue(const mmh3_dims& d, const mmh3_block_weights* w, bool own_mods, const Plan& plan,
                     const Workspace& ws, const float* pos, int n, cudaStream_t s) {
  if (!own_mods && pos == nullptr) return MMH3_OK;
  AdalnBatch ab{};
  if (own_mods) {
    ab.w[0] = w->adaln_w;
    ab.b[0] = w->adaln_b;
    ab.table[0] = w->adaln_table;
  }
  cudaError_t e = launch_prologue(ab, own_mods ? 1 : 0, d.rank, d.grid, 18 * d.hidden, plan, ws.mods, 0, pos, n,
                                  d.rope_k, d.rope_theta, ws.cs, s);
  if (e != cudaSuccess) return cuda_fail(e, "prologue launch");
  return canaries(ws, true, MMH3_PROF_K_PROLOGUE, s);
}

mmh3_status common_checks(const mmh3_dims* dims, float* x, int n, const float* pos, void* ws,
                          size_t ws_bytes, Workspace* out_ws) {
  mmh3_status st = check_dims(dims);
  if (st != MMH3_OK) return st;
  if (x == nullptr) return fail(MMH3_ERR_ARG, "x is null");
  if (misaligned(x) || (pos && misaligned(pos)) || misaligned(ws))
    return fail(MMH3_ERR_ALIGN, "x / pos / workspace must be 16-byte aligned");
  if (n < 1) return fail(MMH3_ERR_SHAPE, "n = %d < 1", n);
  if (fault_injected("workspace")) return fail(MMH3_ERR_WORKSPACE, "injected fault at workspace");
  const Workspace need = carve(*dims, n, nullptr);
  if (ws == nullptr || ws_bytes < need.bytes)
    return fail(MMH3_ERR_WORKSPACE, "workspace %zu bytes < %zu required", ws_bytes, need.bytes);
  *out_ws = carve(*dims, n, ws);
  return MMH3_OK;
}

}  // namespace

// The whole modulated (or unmodulated) block on a caller-provided scratch
// region; shared by the entry points that take a workspace and by the one
// that uses the library's own static scratch.  `profile` = false records no
// phase events.
mmh3_status mmh3::block_forward_impl(const mmh3_dims* dims, const mmh3_block_weights* w, float* x, int n,
                                     const mmh3_segment* segs, int n_seg, const float* pos_dev, double sigma_v,
                                     double sigma_a, int modulated, const float* mods_or_null, void* workspace,
                                     size_t ws_bytes, void* stream, bool profile) {
  Workspace ws;
  mmh3_status st = common_checks(dims, x, n, pos_dev, workspace, ws_bytes, &ws);
  if (st != MMH3_OK) return st;
  // with the caller's modulation the block reads no adaLN weights
  const bool own_mods = modulated && mods_or_null == nullptr;
  st = check_block(*dims, w, own_mods);
  if (st != MMH3_OK) return st;
  if (mods_or_null != nullptr && !modulated)
    return fail(MMH3_ERR_ARG, "mods_or_null given to an unmodulated block");
  if (mods_or_null != nullptr && misaligned(mods_or_null))
    return fail(MMH3_ERR_ALIGN, "mods_or_null is not 16-byte aligned");
  Plan plan;
  if (modulated) {
    st = make_plan(segs, n_seg, n, sigma_v, sigma_a, &plan);
    if (st != MMH3_OK) return st;
    if (own_mods) {
      st = own_curve_slots(plan);
      if (st != MMH3_OK) return st;
    }
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  PhaseMark pm(s, profile);
  st = canaries(ws, false, 0, s);
  if (st != MMH3_OK) return st;
  st = prologue(*dims, w, own_mods, plan, ws, pos_dev, n, s);
  if (st != MMH3_OK) return st;
  if (own_mods || pos_dev) pm.mark(0, MMH3_PROF_K_PROLOGUE);
  const float* mods = !modulated ? nullptr : (mods_or_null ? mods_or_null : ws.mods);
  return block_core(*dims, *w, x, n, plan, mods, pos_dev ? ws.cs : nullptr, ws, s, pm);
}

extern "C" {


mmh3_status mmh3_workspace_size(const mmh3_dims* dims, int n, size_t* bytes) {
  clear_error();
  mmh3_status st = check_dims(dims);
  if (st != MMH3_OK) return st;
  if (bytes == nullptr) return fail(MMH3_ERR_ARG, "bytes is null");
  if (n < 0) return fail(MMH3_ERR_SHAPE, "n < 0");
  *bytes = carve(*dims, n, nullptr).bytes;
  return MMH3_OK;
}

mmh3_status mmh3_resolve_rows(const mmh3_segment* segs, int n_seg, int n, double sigma_v, double sigma_a,
                              int32_t* rows_dev, void* stream) {
  clear_error();
  if (rows_dev == nullptr) return fail(MMH3_ERR_ARG, "rows is null");
  Plan plan;
  mmh3_status st = make_plan(segs, n_seg, n, sigma_v, sigma_a, &plan);
  if (st != MMH3_OK) return st;
  cudaError_t e = launch_rows(plan.block_rows, n, rows_dev, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MMH3_OK : cuda_fail(e, "rows launch");
}

mmh3_status mmh3_adaln_modulation(const mmh3_dims* dims, const float* w, const float* b, const float* table,
                                  int rows_per_slot, const mmh3_segment* segs, int n_seg, int n,
                                  double sigma_v, double sigma_a, float* out, int* n_ts, void* stream) {
  clear_error();
  if (dims == nullptr || w == nullptr || b == nullptr || table == nullptr || out == nullptr)
    return fail(MMH3_ERR_ARG, "adaln: null pointer");
  if (dims->rank < 1 || dims->rank > 32 || dims->grid < 2) return fail(MMH3_ERR_SHAPE, "adaln: rank/grid");
  if (rows_per_slot < 1) return fail(MMH3_ERR_SHAPE, "adaln: rows_per_slot %d", rows_per_slot);
  if (misaligned(w)) return fail(MMH3_ERR_ALIGN, "adaln: basis not 16-byte aligned");
  Plan plan;
  mmh3_status st = make_plan(segs, n_seg, n, sigma_v, sigma_a, &plan);
  if (st != MMH3_OK) return st;
  if (n_ts) *n_ts = plan.n_ts;
  st = own_curve_slots(plan);
  if (st != MMH3_OK) return st;
  cudaError_t e = launch_adaln(w, b, table, dims->rank, dims->grid, rows_per_slot, plan, out,
                               static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MMH3_OK : cuda_fail(e, "adaln launch");
}

mmh3_status mmh3_prepare_block_weights(const mmh3_dims* dims, const void* fc1_gate_up, void* fc1_interleaved,
                                       void* stream) {
  return mmh3_prepare_fc1(dims, fc1_gate_up, fc1_interleaved, stream);
}

mmh3_status mmh3_prepare_fc1(const mmh3_dims* dims, const void* fc1_gate_up, void* fc1_tiled, void* stream) {
  clear_error();
  mmh3_status st = check_dims(dims);
  if (st != MMH3_OK) return st;
  if (fc1_gate_up == nullptr || fc1_tiled == nullptr || fc1_gate_up == fc1_tiled)
    return fail(MMH3_ERR_ARG, "prepare_fc1: null or aliased pointers");
  if (misaligned(fc1_gate_up) || misaligned(fc1_tiled)) return fail(MMH3_ERR_ALIGN, "prepare_fc1: alignment");
  cudaError_t e = launch_fc1_tile(esize_of(dims->act_dtype), fc1_gate_up, fc1_tiled, dims->ffn, dims->hidden,
                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MMH3_OK : cuda_fail(e, "prepare_fc1 launch");
}

mmh3_status mmh3_block_forward(const mmh3_dims* dims, const mmh3_block_weights* w, float* x, int n,
                               const mmh3_segment* segs, int n_seg, const float* pos_dev, double sigma_v,
                               double sigma_a, int modulated, const float* mods_or_null, void* workspace,
                               size_t ws_bytes, void* stream) {
  clear_error();
  return block_forward_impl(dims, w, x, n, segs, n_seg, pos_dev, sigma_v, sigma_a, modulated, mods_or_null,
                            workspace, ws_bytes, stream, /*profile=*/true);
}

mmh3_status mmh3_stack_forward(const mmh3_dims* dims, const mmh3_block_weights* blocks, int n_blocks,
                               const mmh3_head_weights* heads, float* x, int n, const mmh3_segment* segs,
                               int n_seg, const float* pos_dev, double sigma_v, double sigma_a,
                               float* out_video, float* out_audio, void* workspace, size_t ws_bytes,
                               void* stream) {
  clear_error();
  Workspace ws;
  mmh3_status st = common_checks(dims, x, n, pos_dev, workspace, ws_bytes, &ws);
  if (st != MMH3_OK) return st;
  if (n_blocks < 0 || (n_blocks > 0 && blocks == nullptr)) return fail(MMH3_ERR_ARG, "blocks");
  for (int i = 0; i < n_blocks; ++i) {
    st = check_block(*dims, blocks + i, true);
    if (st != MMH3_OK) return st;
  }
  Plan plan;
  st = make_plan(segs, n_seg, n, sigma_v, sigma_a, &plan);
  if (st != MMH3_OK) return st;
  st = own_curve_slots(plan);
  if (st != MMH3_OK) return st;
  const int H = dims->hidden;
  // output streams: the last video-tag segment and the last audio-tag segment
  int vseg = -1, aseg = -1;
  for (int k = 0; k < n_seg; ++k) {
    if (segs[k].tag == 0) vseg = k;
    if (segs[k].tag == 2) aseg = k;
  }
  if (heads) {
    if (heads->final_norm == nullptr || heads->adaln_w == nullptr || heads->adaln_b == nullptr ||
        heads->adaln_table == nullptr)
      return fail(MMH3_ERR_ARG, "head weights: null pointer");
    if (vseg >= 0 && (heads->w_video == nullptr || heads->b_video == nullptr || out_video == nullptr ||
                      heads->out_video <= 0 || heads->out_video % 32 != 0))
      return fail(MMH3_ERR_ARG, "video head: missing pointer or out_video %d not a positive multiple of 32",
                  heads->out_video);
    if (aseg >= 0 && (heads->w_audio == nullptr || heads->b_audio == nullptr || out_audio == nullptr ||
                      heads->out_audio <= 0 || heads->out_audio % 32 != 0))
      return fail(MMH3_ERR_ARG, "audio head: missing pointer or out_audio %d not a positive multiple of 32",
                  heads->out_audio);
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  PhaseMark pm(s, true);
  // Every block's modulation is evaluated up front, up to kAdalnBatch blocks
  // per launch, into the head-scratch region (unused until the heads); the
  // first launch also writes the rotation table.  When that region cannot
  // hold one block's rows, each block's modulation goes to ws.mods just
  // before the block.
  st = canaries(ws, false, 0, s);
  if (st != MMH3_OK) return st;
  const long long mods_floats = (long long)plan.n_ts * 18 * H;
  const size_t head_bytes = (size_t)n * H * esize_of(dims->act_dtype);
  long long fit = (long long)(head_bytes / ((size_t)mods_floats * 4));
  const int per_launch = (int)std::max(1ll, std::min<long long>(kAdalnBatch, fit));
  float* mbase = fit >= 1 ? static_cast<float*>(ws.head) : ws.mods;
  if (n_blocks == 0 && pos_dev) {
    cudaError_t e = launch_prologue(AdalnBatch{}, 0, dims->rank, dims->grid, 18 * H, plan, mbase, mods_floats,
                                    pos_dev, n, dims->rope_k, dims->rope_theta, ws.cs, s);
    if (e != cudaSuccess) return cuda_fail(e, "prologue launch");
    pm.mark(0, MMH3_PROF_K_PROLOGUE);
    st = canaries(ws, true, MMH3_PROF_K_PROLOGUE, s);
    if (st != MMH3_OK) return st;
  }
  for (int i = 0; i < n_blocks; ++i) {
    if (i % per_launch == 0) {
      const int cnt = std::min(per_launch, n_blocks - i);
      AdalnBatch ab{};
      for (int b = 0; b < cnt; ++b) {
        ab.w[b] = blocks[i + b].adaln_w;
        ab.b[b] = blocks[i + b].adaln_b;
        ab.table[b] = blocks[i + b].adaln_table;
      }
      cudaError_t e = launch_prologue(ab, cnt, dims->rank, dims->grid, 18 * H, plan, mbase, mods_floats,
                                      i == 0 ? pos_dev : nullptr, n, dims->rope_k, dims->rope_theta, ws.cs, s);
      if (e != cudaSuccess) return cuda_fail(e, "prologue launch");
      pm.mark(0, MMH3_PROF_K_PROLOGUE);
      st = canaries(ws, true, MMH3_PROF_K_PROLOGUE, s);
      if (st != MMH3_OK) return st;
    }
    const float* mods = mbase + (i % per_launch) * mods_floats;
    st = block_core(*dims, blocks[i], x, n, plan, mods, pos_dev ? ws.cs : nullptr, ws, s, pm);
    if (st != MMH3_OK) return st;
  }
  if (heads == nullptr) return MMH3_OK;
  cudaError_t e = launch_adaln(heads->adaln_w, heads->adaln_b, heads->adaln_table, dims->rank, dims->grid, 2 * H,
                               plan, ws.fmods, s);
  if (e != cudaSuccess) return cuda_fail(e, "final adaln launch");
  const int sidx[2] = {vseg, aseg};
  for (int k = 0; k < 2; ++k) {
    if (sidx[k] < 0) continue;
    const mmh3_segment& sg = segs[sidx[k]];
    const int rows = (int)(sg.stop - sg.start);
    e = launch_norm_mod(dims->act_dtype, x + (size_t)sg.start * H, rows, H, heads->final_norm, dims->eps,
                        ws.fmods, 2 * H, 0, H, plan.final_rows, (int)sg.start, ws.head, s);
    if (e != cudaSuccess) return cuda_fail(e, "final norm launch");
    st = gemm_bias_act(dims->act_dtype, ws.head, k == 0 ? heads->w_video : heads->w_audio, rows,
                       k == 0 ? heads->out_video : heads->out_audio, H, k == 0 ? heads->b_video : heads->b_audio, 2,
                       k == 0 ? (void*)out_video : (void*)out_audio, s);
    if (st != MMH3_OK) return st;
    st = canaries(ws, true, 8, s);
    if (st != MMH3_OK) return st;
  }
  return MMH3_OK;
}

// ----------------------------------------------- block on host buffers
namespace {

// Per device: the events that order the copy-in, compute and copy-out
// streams of the staging slots.
struct HostSlots {
  bool ready = false;
  cudaEvent_t in_done[MMH3_HOST_SLOTS], compute_done[MMH3_HOST_SLOTS], out_done[MMH3_HOST_SLOTS];
};
constexpr int kMaxHostDevices = 64;
HostSlots g_host_slots[kMaxHostDevices];
std::mutex g_host_mu;

mmh3_status host_slots(HostSlots** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "host pipeline: cudaGetDevice");
  if (dev < 0 || dev >= kMaxHostDevices) return fail(MMH3_ERR_UNSUPPORTED, "host pipeline: device %d", dev);
  std::lock_guard<std::mutex> lock(g_host_mu);
  HostSlots& h = g_host_slots[dev];
  if (!h.ready) {
    for (int k = 0; k < MMH3_HOST_SLOTS; ++k) {
      cudaEvent_t* evs[3] = {&h.in_done[k], &h.compute_done[k], &h.out_done[k]};
      for (cudaEvent_t* ev : evs) {
        e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
        if (e != cudaSuccess) return cuda_fail(e, "host pipeline: event");
      }
      // a never-used slot counts as free: record the "copied out" event once
      e = cudaEventRecord(h.out_done[k], 0);
      if (e != cudaSuccess) return cuda_fail(e, "host pipeline: event record");
    }
    h.ready = true;
  }
  *out = &h;
  return MMH3_OK;
}

}  // namespace

mmh3_status mmh3_block_forward_host(const mmh3_dims* dims, const mmh3_block_weights* w, const float* x_in_host,
                                    float* x_out_host, int n, const mmh3_segment* segs, int n_seg,
                                    const float* pos_host, double sigma_v, double sigma_a, int slot,
                                    float* x_dev, float* pos_dev, void* workspace, size_t ws_bytes, void* stream,
                                    void* copy_in_stream, void* copy_out_stream) {
  clear_error();
  mmh3_status st = check_dims(dims);
  if (st != MMH3_OK) return st;
  if (slot < 0 || slot >= MMH3_HOST_SLOTS)
    return fail(MMH3_ERR_ARG, "host block: slot %d outside [0, %d)", slot, MMH3_HOST_SLOTS);
  if (!x_in_host || !x_out_host || !x_dev) return fail(MMH3_ERR_ARG, "host block: null x buffer");
  if ((pos_host == nullptr) != (pos_dev == nullptr))
    return fail(MMH3_ERR_ARG, "host block: pos_host and pos_dev must both be given or both be null");
  if (n < 1) return fail(MMH3_ERR_SHAPE, "host block: n = %d < 1", n);
  HostSlots* h = nullptr;
  st = host_slots(&h);
  if (st != MMH3_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaStream_t si = static_cast<cudaStream_t>(copy_in_stream);
  cudaStream_t so = static_cast<cudaStream_t>(copy_out_stream);
  const size_t xb = (size_t)n * dims->hidden * sizeof(float), pb = (size_t)n * 3 * sizeof(float);
  // 1. copy in, once the slot's previous result has left the device
  cudaError_t e = cudaStreamWaitEvent(si, h->out_done[slot], 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(x_dev, x_in_host, xb, cudaMemcpyHostToDevice, si);
  if (e == cudaSuccess && pos_host) e = cudaMemcpyAsync(pos_dev, pos_host, pb, cudaMemcpyHostToDevice, si);
  if (e == cudaSuccess) e = cudaEventRecord(h->in_done[slot], si);
  if (e != cudaSuccess) return cuda_fail(e, "host block: copy in");
  // 2. the block, after its input arrived
  e = cudaStreamWaitEvent(s, h->in_done[slot], 0);
  if (e != cudaSuccess) return cuda_fail(e, "host block: wait for the input");
  st = mmh3::block_forward_impl(dims, w, x_dev, n, segs, n_seg, pos_dev, sigma_v, sigma_a, 1, nullptr, workspace,
                                ws_bytes, stream, /*profile=*/false);
  if (st != MMH3_OK) return st;
  e = cudaEventRecord(h->compute_done[slot], s);
  // 3. copy the result out
  if (e == cudaSuccess) e = cudaStreamWaitEvent(so, h->compute_done[slot], 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(x_out_host, x_dev, xb, cudaMemcpyDeviceToHost, so);
  if (e == cudaSuccess) e = cudaEventRecord(h->out_done[slot], so);
  return e == cudaSuccess ? MMH3_OK : cuda_fail(e, "host block: copy out");
}

// ------------------------------------------- block over a sequence shard
mmh3_status mmh3_block_cp_begin(const mmh3_dims* dims, const mmh3_block_weights* w, const float* x, int n,
                                const mmh3_segment* segs, int n_seg, const float* pos_dev, double sigma_v,
                                double sigma_a, int modulated, void* kv_out, void* workspace, size_t ws_bytes,
                                void* stream) {
  clear_error();
  Workspace ws;
  mmh3_status st = common_checks(dims, const_cast<float*>(x), n, pos_dev, workspace, ws_bytes, &ws);
  if (st != MMH3_OK) return st;
  if (dims->act_dtype != MMH3_BF16) return fail(MMH3_ERR_UNSUPPORTED, "sequence shards: bf16 activations only");
  if (kv_out == nullptr || misaligned(kv_out)) return fail(MMH3_ERR_ARG, "kv_out null or not 16-byte aligned");
  st = check_block(*dims, w, modulated != 0);
  if (st != MMH3_OK) return st;
  Plan plan;
  if (modulated) {
    st = make_plan(segs, n_seg, n, sigma_v, sigma_a, &plan);
    if (st != MMH3_OK) return st;
    st = own_curve_slots(plan);
    if (st != MMH3_OK) return st;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  PhaseMark pm(s, false);
  st = canaries(ws, false, 0, s);
  if (st != MMH3_OK) return st;
  st = prologue(*dims, w, modulated != 0, plan, ws, pos_dev, n, s);
  if (st != MMH3_OK) return st;
  st = block_pre(*dims, *w, x, n, plan, modulated ? ws.mods : nullptr, pos_dev ? ws.cs : nullptr, ws, s, pm);
  if (st != MMH3_OK) return st;
  const size_t I = (size_t)dims->heads * dims->head_dim;
  cudaError_t e = cudaMemcpy2DAsync(kv_out, 2 * I * 2, static_cast<const uint8_t*>(ws.qkv) + I * 2, 3 * I * 2,
                                    2 * I * 2, (size_t)n, cudaMemcpyDeviceToDevice, s);
  return e == cudaSuccess ? MMH3_OK : cuda_fail(e, "K|V export copy");
}

mmh3_status mmh3_block_cp_end(const mmh3_dims* dims, const mmh3_block_weights* w, float* x, int n,
                              const mmh3_segment* segs, int n_seg, double sigma_v, double sigma_a, int modulated,
                              const void* kv_all, int n_kv, void* workspace, size_t ws_bytes, void* stream) {
  clear_error();
  Workspace ws;
  mmh3_status st = common_checks(dims, x, n, nullptr, workspace, ws_bytes, &ws);
  if (st != MMH3_OK) return st;
  if (dims->act_dtype != MMH3_BF16) return fail(MMH3_ERR_UNSUPPORTED, "sequence shards: bf16 activations only");
  if (kv_all == nullptr || misaligned(kv_all)) return fail(MMH3_ERR_ARG, "kv_all null or not 16-byte aligned");
  if (n_kv < n) return fail(MMH3_ERR_SHAPE, "n_kv = %d keys < the shard's %d rows", n_kv, n);
  st = check_block(*dims, w, modulated != 0);
  if (st != MMH3_OK) return st;
  Plan plan;
  if (modulated) {
    st = make_plan(segs, n_seg, n, sigma_v, sigma_a, &plan);
    if (st != MMH3_OK) return st;
    st = own_curve_slots(plan);
    if (st != MMH3_OK) return st;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  PhaseMark pm(s, false);
  return block_post(*dims, *w, x, n, plan, modulated ? ws.mods : nullptr, ws, s, pm, kv_all, n_kv);
}

// ------------------------------------------------------------ token refiner
static size_t refine_stream_offset(const mmh3_dims& d, int n) { return carve(d, n, nullptr).bytes; }

mmh3_status mmh3_refine_workspace_size(const mmh3_dims* dims, int n, size_t* bytes) {
  clear_error();
  mmh3_status st = check_dims(dims);
  if (st != MMH3_OK) return st;
  if (bytes == nullptr || n < 0) return fail(MMH3_ERR_ARG, "refine workspace: bytes null or n < 0");
  *bytes = refine_stream_offset(*dims, n) + align256((size_t)n * dims->hidden * 4);
  return MMH3_OK;
}

mmh3_status mmh3_refine_text(const mmh3_dims* dims, const void* states, int n, int text_dim, const void* cond_w,
                             const float* cond_b, const mmh3_block_weights* blocks, int n_blocks,
                             const float* refiner_norm, float final_eps, float* out, void* workspace,
                             size_t ws_bytes, void* stream) {
  clear_error();
  mmh3_status st = check_dims(dims);
  if (st != MMH3_OK) return st;
  if (!states || !cond_w || !cond_b || !refiner_norm || !out || !workspace)
    return fail(MMH3_ERR_ARG, "refine: null pointer");
  if (misaligned(states) || misaligned(cond_w) || misaligned(cond_b) || misaligned(refiner_norm) ||
      misaligned(out) || misaligned(workspace))
    return fail(MMH3_ERR_ALIGN, "refine: pointers must be 16-byte aligned");
  if (n < 1) return fail(MMH3_ERR_SHAPE, "refine: n = %d < 1", n);
  const int es = esize_of(dims->act_dtype);
  if (text_dim < 1 || ((size_t)text_dim * es) % 16 != 0)
    return fail(MMH3_ERR_SHAPE, "refine: text_dim %d * %d bytes not a positive multiple of 16", text_dim, es);
  if (!(final_eps > 0)) return fail(MMH3_ERR_ARG, "refine: final_eps must be positive");
  if (n_blocks < 0 || (n_blocks > 0 && blocks == nullptr)) return fail(MMH3_ERR_ARG, "refine: blocks");
  for (int i = 0; i < n_blocks; ++i) {
    st = check_block(*dims, blocks + i, false);
    if (st != MMH3_OK) return st;
  }
  size_t need = 0;
  mmh3_refine_workspace_size(dims, n, &need);
  if (ws_bytes < need) return fail(MMH3_ERR_WORKSPACE, "refine workspace %zu bytes < %zu required", ws_bytes, need);
  const Workspace ws = carve(*dims, n, workspace);
  float* h = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + refine_stream_offset(*dims, n));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int H = dims->hidden;
  st = canaries(ws, false, 0, s);
  if (st != MMH3_OK) return st;
  st = gemm_bias_act(dims->act_dtype, states, cond_w, n, H, text_dim, cond_b, 3, h, s);
  if (st != MMH3_OK) return st;
  PhaseMark pm(s, false);
  const Plan plan{};
  for (int i = 0; i < n_blocks; ++i) {
    st = block_core(*dims, blocks[i], h, n, plan, nullptr, nullptr, ws, s, pm);
    if (st != MMH3_OK) return st;
  }
  cudaError_t e = launch_norm_mod(MMH3_F32, h, n, H, refiner_norm, final_eps, nullptr, 0, 0, 0, SegRows{}, 0, out, s);
  return e == cudaSuccess ? MMH3_OK : cuda_fail(e, "refiner final norm launch");
}

// ------------------------------------------------------------------- embed
namespace {

struct StreamShape {
  long rows;
  int K;
};

mmh3_status stream_shape(int kind, int C, int T, int lh, int lw, StreamShape* out) {
  if (C < 1 || T < 0) return fail(MMH3_ERR_SHAPE, "stream: channels %d frames %d", C, T);
  if (kind == MMH3_STREAM_VIDEO) {
    if (lh < 2 || lw < 2 || (lh & 1) || (lw & 1))
      return fail(MMH3_ERR_SHAPE, "video latents %d x %d: both sides must be even and >= 2", lh, lw);
    out->rows = (long)T * (lh / 2) * (lw / 2);
    out->K = 4 * C;
    return MMH3_OK;
  }
  if (kind == MMH3_STREAM_AUDIO) {
    out->rows = 2L * T;
    out->K = C;
    return MMH3_OK;
  }
  return fail(MMH3_ERR_ARG, "stream kind %d is neither video (0) nor audio (2)", kind);
}

}  // namespace

mmh3_status mmh3_patch_embed_workspace_size(const mmh3_dims* dims, int kind, int channels, int frames, int lat_h,
                                            int lat_w, size_t* bytes) {
  clear_error();
  mmh3_status st = check_dims(dims);
  if (st != MMH3_OK) return st;
  if (bytes == nullptr) return fail(MMH3_ERR_ARG, "patch embed workspace: bytes null");
  StreamShape sh;
  st = stream_shape(kind, channels, frames, lat_h, lat_w, &sh);
  if (st != MMH3_OK) return st;
  *bytes = align256((size_t)sh.rows * sh.K * esize_of(dims->act_dtype));
  return MMH3_OK;
}

mmh3_status mmh3_patch_embed(const mmh3_dims* dims, int kind, const float* latents, int channels, int frames,
                             int lat_h, int lat_w, const void* w, const float* b, float* x_rows, void* workspace,
                             size_t ws_bytes, void* stream) {
  clear_error();
  size_t need = 0;
  mmh3_status st = mmh3_patch_embed_workspace_size(dims, kind, channels, frames, lat_h, lat_w, &need);
  if (st != MMH3_OK) return st;
  StreamShape sh;
  stream_shape(kind, channels, frames, lat_h, lat_w, &sh);
  if (sh.rows == 0) return MMH3_OK;
  if (!latents || !w || !b || !x_rows || !workspace) return fail(MMH3_ERR_ARG, "patch embed: null pointer");
  if (misaligned(w) || misaligned(b) || misaligned(x_rows) || misaligned(workspace))
    return fail(MMH3_ERR_ALIGN, "patch embed: w / b / x_rows / workspace must be 16-byte aligned");
  const int es = esize_of(dims->act_dtype);
  if (((size_t)sh.K * es) % 16 != 0)
    return fail(MMH3_ERR_SHAPE, "patch embed: K = %d * %d bytes is not a multiple of 16", sh.K, es);
  if (sh.rows > INT32_MAX) return fail(MMH3_ERR_SHAPE, "patch embed: %ld rows", sh.rows);
  if (ws_bytes < need) return fail(MMH3_ERR_WORKSPACE, "patch embed workspace %zu < %zu", ws_bytes, need);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = kind == MMH3_STREAM_VIDEO
                      ? launch_patchify(dims->act_dtype, latents, channels, frames, lat_h, lat_w, workspace, s)
                      : launch_pack_audio(dims->act_dtype, latents, channels, frames, workspace, s);
  if (e != cudaSuccess) return cuda_fail(e, "patchify / pack launch");
  return gemm_bias_act(dims->act_dtype, workspace, w, (int)sh.rows, dims->hidden, sh.K, b, 3, x_rows, s);
}

mmh3_status mmh3_embed_workspace_size(const mmh3_dims* dims, const mmh3_embed_inputs* in, size_t* bytes) {
  clear_error();
  if (in == nullptr || bytes == nullptr) return fail(MMH3_ERR_ARG, "embed workspace: null");
  size_t v = 0, c = 0, a = 0;
  mmh3_status st = mmh3_patch_embed_workspace_size(dims, MMH3_STREAM_VIDEO, in->video_channels, in->video_frames,
                                                   in->lat_h, in->lat_w, &v);
  if (st != MMH3_OK) return st;
  st = mmh3_patch_embed_workspace_size(dims, MMH3_STREAM_VIDEO, in->video_channels, 1, in->lat_h, in->lat_w, &c);
  if (st != MMH3_OK) return st;
  st = mmh3_patch_embed_workspace_size(dims, MMH3_STREAM_AUDIO, in->audio_channels, in->audio_frames, 0, 0, &a);
  if (st != MMH3_OK) return st;
  *bytes = std::max(v, std::max(in->n_cond > 0 ? c : (size_t)0, a));
  return MMH3_OK;
}

mmh3_status mmh3_embed(const mmh3_dims* dims, const mmh3_segment* segs, int n_seg, int n,
                       const mmh3_embed_inputs* in, const mmh3_embed_weights* w, float* x, void* workspace,
                       size_t ws_bytes, void* stream) {
  clear_error();
  if (in == nullptr || w == nullptr || x == nullptr || segs == nullptr)
    return fail(MMH3_ERR_ARG, "embed: null pointer");
  mmh3_status st = check_dims(dims);
  if (st != MMH3_OK) return st;
  Plan plan;
  st = make_plan(segs, n_seg, n, 0.5, 0.5, &plan);  // validates the segment table only
  if (st != MMH3_OK) return st;
  int t_seg = -1, a_seg = -1, v_last = -1, n_other = 0;
  for (int k = 0; k < n_seg; ++k) {
    if (segs[k].clock == 3)
      return fail(MMH3_ERR_UNSUPPORTED, "embed: segment %d holds reference audio, which has no input here", k);
    if (segs[k].tag == 1 && t_seg < 0) t_seg = k;
    if (segs[k].tag == 2) a_seg = k;
    if (segs[k].tag == 0) v_last = k;
  }
  for (int k = 0; k < v_last; ++k) n_other += segs[k].tag == 0;
  if (in->n_cond != n_other || (n_other > 0 && in->cond == nullptr))
    return fail(MMH3_ERR_ARG, "embed: %d condition frames given, the segments hold %d", in->n_cond, n_other);
  const size_t H = (size_t)dims->hidden;
  const long frame_rows = (long)(in->lat_h / 2) * (in->lat_w / 2);
  if (v_last >= 0 && (long)(segs[v_last].stop - segs[v_last].start) != frame_rows * in->video_frames)
    return fail(MMH3_ERR_SHAPE, "embed: video segment of %u rows, the latents give %ld",
                segs[v_last].stop - segs[v_last].start, frame_rows * in->video_frames);
  if (a_seg >= 0 && (long)(segs[a_seg].stop - segs[a_seg].start) != 2L * in->audio_frames)
    return fail(MMH3_ERR_SHAPE, "embed: audio segment of %u rows, the latents give %d",
                segs[a_seg].stop - segs[a_seg].start, 2 * in->audio_frames);
  for (int k = 0; k < v_last; ++k)
    if (segs[k].tag == 0 && (long)(segs[k].stop - segs[k].start) != frame_rows)
      return fail(MMH3_ERR_SHAPE, "embed: condition segment %d of %u rows, a frame gives %ld", k,
                  segs[k].stop - segs[k].start, frame_rows);
  if (t_seg >= 0 && in->text == nullptr) return fail(MMH3_ERR_ARG, "embed: text is null");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (t_seg >= 0) {
    const size_t rows = segs[t_seg].stop - segs[t_seg].start;
    cudaError_t e = cudaMemcpyAsync(x + segs[t_seg].start * H, in->text, rows * H * sizeof(float),
                                    cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "embed: text copy");
  }
  if (v_last >= 0) {
    st = mmh3_patch_embed(dims, MMH3_STREAM_VIDEO, in->video, in->video_channels, in->video_frames, in->lat_h,
                          in->lat_w, w->w_video, w->b_video, x + segs[v_last].start * H, workspace, ws_bytes, s);
    if (st != MMH3_OK) return st;
  }
  for (int k = 0, ci = 0; k < v_last; ++k) {
    if (segs[k].tag != 0) continue;
    st = mmh3_patch_embed(dims, MMH3_STREAM_VIDEO, in->cond[ci++], in->video_channels, 1, in->lat_h, in->lat_w,
                          w->w_video, w->b_video, x + segs[k].start * H, workspace, ws_bytes, s);
    if (st != MMH3_OK) return st;
  }
  if (a_seg >= 0) {
    st = mmh3_patch_embed(dims, MMH3_STREAM_AUDIO, in->audio, in->audio_channels, in->audio_frames, 0, 0,
                          w->w_audio, w->b_audio, x + segs[a_seg].start * H, workspace, ws_bytes, s);
    if (st != MMH3_OK) return st;
  }
  return MMH3_OK;
}

mmh3_status mmh3_unpatchify_video(const float* rows, int channels, int frames, int lat_h, int lat_w, float* out,
                                  void* stream) {
  clear_error();
  StreamShape sh;
  mmh3_status st = stream_shape(MMH3_STREAM_VIDEO, channels, frames, lat_h, lat_w, &sh);
  if (st != MMH3_OK) return st;
  if (sh.rows == 0) return MMH3_OK;
  if (rows == nullptr || out == nullptr) return fail(MMH3_ERR_ARG, "unpatchify: null pointer");
  cudaError_t e = launch_unpatchify(rows, channels, frames, lat_h, lat_w, out, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MMH3_OK : cuda_fail(e, "unpatchify launch");
}

mmh3_status mmh3_unpack_audio(const float* rows, int channels, int frames, float* out, void* stream) {
  clear_error();
  if (channels < 1 || frames < 0) return fail(MMH3_ERR_SHAPE, "unpack audio: channels %d frames %d", channels, frames);
  if (frames == 0) return MMH3_OK;
  if (rows == nullptr || out == nullptr) return fail(MMH3_ERR_ARG, "unpack audio: null pointer");
  cudaError_t e = launch_unpack_audio(rows, channels, frames, out, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MMH3_OK : cuda_fail(e, "unpack audio launch");
}

// ------------------------------------------------- one denoise evaluation
namespace {

struct ForwardCarve {
  size_t stage, video_rows, audio_rows, bytes;
};

mmh3_status forward_carve(const mmh3_dims* dims, int n, const mmh3_embed_inputs* in, ForwardCarve* c) {
  size_t emb = 0;
  mmh3_status st = mmh3_embed_workspace_size(dims, in, &emb);
  if (st != MMH3_OK) return st;
  const size_t stack = carve(*dims, n, nullptr).bytes;
  const size_t nv = (size_t)in->video_frames * (in->lat_h / 2) * (in->lat_w / 2);
  c->stage = std::max(stack, emb);
  c->video_rows = c->stage;
  c->audio_rows = c->video_rows + align256(nv * 4 * in->video_channels * sizeof(float));
  c->bytes = c->audio_rows + align256(2 * (size_t)in->audio_frames * in->audio_channels * sizeof(float));
  return MMH3_OK;
}

}  // namespace

mmh3_status mmh3_forward_workspace_size(const mmh3_dims* dims, int n, const mmh3_embed_inputs* in, size_t* bytes) {
  clear_error();
  mmh3_status st = check_dims(dims);
  if (st != MMH3_OK) return st;
  if (in == nullptr || bytes == nullptr || n < 1) return fail(MMH3_ERR_ARG, "forward workspace: null or n < 1");
  ForwardCarve c;
  st = forward_carve(dims, n, in, &c);
  if (st != MMH3_OK) return st;
  *bytes = c.bytes;
  return MMH3_OK;
}

mmh3_status mmh3_forward(const mmh3_dims* dims, const mmh3_segment* segs, int n_seg, int n, const float* pos_dev,
                         double sigma_v, double sigma_a, const mmh3_embed_inputs* in, const mmh3_embed_weights* ew,
                         const mmh3_block_weights* blocks, int n_blocks, const mmh3_head_weights* heads, float* x,
                         float* video_out, float* audio_out, void* workspace, size_t ws_bytes, void* stream) {
  clear_error();
  if (heads == nullptr || in == nullptr || ew == nullptr || segs == nullptr)
    return fail(MMH3_ERR_ARG, "forward: null heads / inputs / weights / segments");
  size_t need = 0;
  mmh3_status st = mmh3_forward_workspace_size(dims, n, in, &need);
  if (st != MMH3_OK) return st;
  if (workspace == nullptr || ws_bytes < need)
    return fail(MMH3_ERR_WORKSPACE, "forward workspace %zu bytes < %zu required", ws_bytes, need);
  bool has_v = false, has_a = false;
  for (int k = 0; k < n_seg && k < 64; ++k) {
    has_v |= segs[k].tag == 0;
    has_a |= segs[k].tag == 2;
  }
  if (has_v && (heads->out_video != 4 * in->video_channels || video_out == nullptr))
    return fail(MMH3_ERR_SHAPE, "forward: video head width %d != 4 * %d latent channels, or video_out null",
                heads->out_video, in->video_channels);
  if (has_a && (heads->out_audio != in->audio_channels || audio_out == nullptr))
    return fail(MMH3_ERR_SHAPE, "forward: audio head width %d != %d latent channels, or audio_out null",
                heads->out_audio, in->audio_channels);
  ForwardCarve c;
  forward_carve(dims, n, in, &c);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  float* vrows = reinterpret_cast<float*>(base + c.video_rows);
  float* arows = reinterpret_cast<float*>(base + c.audio_rows);
  st = mmh3_embed(dims, segs, n_seg, n, in, ew, x, workspace, c.stage, stream);
  if (st != MMH3_OK) return st;
  st = mmh3_stack_forward(dims, blocks, n_blocks, heads, x, n, segs, n_seg, pos_dev, sigma_v, sigma_a, vrows, arows,
                          workspace, c.stage, stream);
  if (st != MMH3_OK) return st;
  if (has_v) {
    st = mmh3_unpatchify_video(vrows, in->video_channels, in->video_frames, in->lat_h, in->lat_w, video_out, stream);
    if (st != MMH3_OK) return st;
  }
  if (has_a) return mmh3_unpack_audio(arows, in->audio_channels, in->audio_frames, audio_out, stream);
  return MMH3_OK;
}

// ----------------------------------------------------------- encoder layer
static mmh3_status check_vit(const mmh3_vit_dims* d) {
  if (d == nullptr) return fail(MMH3_ERR_ARG, "vit dims null");
  if (d->hidden <= 0 || d->hidden % 256 != 0 || d->hidden > 4096)
    return fail(MMH3_ERR_SHAPE, "vit hidden %d must be a multiple of 256", d->hidden);
  if (d->head_dim != 64 && d->head_dim != 128) return fail(MMH3_ERR_SHAPE, "vit head_dim %d", d->head_dim);
  if (d->heads * d->head_dim != d->hidden) return fail(MMH3_ERR_SHAPE, "vit heads*head_dim != hidden");
  if (d->mlp <= 0 || d->mlp % 256 != 0) return fail(MMH3_ERR_SHAPE, "vit mlp %d must be a multiple of 256", d->mlp);
  if (!(d->ln_eps > 0)) return fail(MMH3_ERR_ARG, "vit ln_eps");
  return MMH3_OK;
}

static size_t vit_carve(const mmh3_vit_dims& d, size_t rows, void* base, void** h, void** qkv, void** attn,
                        void** act, void** sched) {
  size_t off = 0;
  auto take = [&](size_t bytes) {
    void* p = base ? static_cast<void*>(static_cast<uint8_t*>(base) + off) : nullptr;
    off += align256(bytes);
    return p;
  };
  *h = take(rows * d.hidden * 2);
  *qkv = take(rows * 3 * d.hidden * 2);
  *attn = take(rows * d.hidden * 2);
  *act = take(rows * d.mlp * 2);
  *sched = take(16);
  return off;
}

mmh3_status mmh3_vit_workspace_size(const mmh3_vit_dims* dims, int batch, int seq, size_t* bytes) {
  clear_error();
  mmh3_status st = check_vit(dims);
  if (st != MMH3_OK) return st;
  if (bytes == nullptr || batch < 0 || seq < 0) return fail(MMH3_ERR_ARG, "vit workspace args");
  void *a, *b, *c, *e, *f;
  *bytes = vit_carve(*dims, (size_t)batch * seq, nullptr, &a, &b, &c, &e, &f);
  return MMH3_OK;
}

mmh3_status mmh3_vit_fold_qkv(const mmh3_vit_dims* dims, const void* wq, const void* wk, const void* wv,
                              const float* bq, const float* bk, const float* bv, void* wqkv, float* bqkv,
                              void* stream) {
  clear_error();
  mmh3_status st = check_vit(dims);
  if (st != MMH3_OK) return st;
  if (!wq || !wk || !wv || !bq || !bk || !bv || !wqkv || !bqkv) return fail(MMH3_ERR_ARG, "vit fold: null");
  const float scale = 1.0f / std::sqrt((float)dims->head_dim);
  cudaError_t e = launch_vit_fold(wq, wk, wv, bq, bk, bv, scale, dims->hidden, wqkv, bqkv,
                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MMH3_OK : cuda_fail(e, "vit fold launch");
}

mmh3_status mmh3_vit_layer_forward(const mmh3_vit_dims* dims, const mmh3_vit_weights* w, float* x, int batch,
                                   int seq, void* workspace, size_t ws_bytes, void* stream) {
  clear_error();
  mmh3_status st = check_vit(dims);
  if (st != MMH3_OK) return st;
  if (w == nullptr || x == nullptr) return fail(MMH3_ERR_ARG, "vit: null pointer");
  const void* req[] = {w->ln1_g, w->ln1_b, w->wqkv, w->bqkv, w->wo, w->bo, w->ln2_g, w->ln2_b, w->w1, w->b1, w->w2, w->b2};
  for (const void* p : req) {
    if (p == nullptr) return fail(MMH3_ERR_ARG, "vit: null weight pointer");
    if (misaligned(p)) return fail(MMH3_ERR_ALIGN, "vit: weight pointer not 16-byte aligned");
  }
  if (batch < 1 || seq < 1) return fail(MMH3_ERR_SHAPE, "vit: batch %d seq %d", batch, seq);
  if (misaligned(x) || misaligned(workspace)) return fail(MMH3_ERR_ALIGN, "vit: x / workspace alignment");
  void *h, *qkv, *attn, *act, *sched;
  const size_t rows = (size_t)batch * seq;
  const size_t need = vit_carve(*dims, rows, nullptr, &h, &qkv, &attn, &act, &sched);
  if (workspace == nullptr || ws_bytes < need)
    return fail(MMH3_ERR_WORKSPACE, "vit workspace %zu < %zu", ws_bytes, need);
  vit_carve(*dims, rows, workspace, &h, &qkv, &attn, &act, &sched);
  unsigned* ticket = static_cast<unsigned*>(sched);  // attention's work counter, zeroed by LN1
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int H = dims->hidden, M = (int)rows;
  // profiler slots as the block's: LayerNorm in the norm slot, the four
  // projections in the GEMM slots, attention in its own
  PhaseMark pm(s, true);
  cudaError_t e =
      launch_layernorm(x, M, H, w->ln1_g, w->ln1_b, dims->ln_eps, static_cast<__nv_bfloat16*>(h), s, ticket);
  if (e != cudaSuccess) return cuda_fail(e, "ln1 launch");
  pm.mark(0, MMH3_PROF_K_NORM1);
  st = gemm_bias_act(MMH3_BF16, h, w->wqkv, M, 3 * H, H, w->bqkv, 0, qkv, s);
  if (st != MMH3_OK) return st;
  pm.mark(1, MMH3_PROF_K_QKV);
  // h is free between the qkv projection and LN2: it holds the partial
  // results of split attention units
  st = attention(MMH3_BF16, qkv, batch, seq, dims->heads, dims->head_dim, 1.0f, attn, s, h, rows * H * 2, ticket);
  if (st != MMH3_OK) return st;
  pm.mark(3, MMH3_PROF_K_ATTN);
  st = gemm_bias_residual(MMH3_BF16, attn, w->wo, M, H, H, w->bo, x, s);
  if (st != MMH3_OK) return st;
  pm.mark(4, MMH3_PROF_K_OUT);
  e = launch_layernorm(x, M, H, w->ln2_g, w->ln2_b, dims->ln_eps, static_cast<__nv_bfloat16*>(h), s);
  if (e != cudaSuccess) return cuda_fail(e, "ln2 launch");
  pm.mark(0, MMH3_PROF_K_NORM2);
  st = gemm_bias_act(MMH3_BF16, h, w->w1, M, dims->mlp, H, w->b1, 1, act, s);
  if (st != MMH3_OK) return st;
  pm.mark(5, MMH3_PROF_K_FC1);
  st = gemm_bias_residual(MMH3_BF16, act, w->w2, M, H, dims->mlp, w->b2, x, s);
  if (st != MMH3_OK) return st;
  pm.mark(7, MMH3_PROF_K_FC2);
  if (pm.on) ++g_prof_blocks;
  return MMH3_OK;
}

// ---------------------------------------------------------------- profiler
void mmh3_prof_enable(int on) { g_prof_on = on != 0; }

mmh3_status mmh3_prof_collect(double* ms, int n_slots, long* n_blocks) {
  clear_error();
  for (ProfRec& r : g_prof_recs) {
    float t = 0.f;
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t, r.a, r.b);
    if (e != cudaSuccess) return cuda_fail(e, "prof: event");
    g_prof_ms[r.slot] += t;
    if (r.kernel >= 0 && r.kernel < MMH3_PROF_KERNELS) {
      g_prof_kms[r.kernel] += t;
      ++g_prof_kcalls[r.kernel];
    }
    g_prof_free.push_back(r.a);
    g_prof_free.push_back(r.b);
  }
  g_prof_recs.clear();
  for (int i = 0; i < n_slots && i < 9; ++i) ms[i] = g_prof_ms[i];
  if (n_blocks) *n_blocks = g_prof_blocks;
  return MMH3_OK;
}

mmh3_status mmh3_prof_collect_kernels(double* ms, long* calls, int n_kernels) {
  clear_error();
  if (n_kernels < 0 || (n_kernels > 0 && ms == nullptr)) return fail(MMH3_ERR_ARG, "prof: ms is null");
  double phases[9];
  mmh3_status st = mmh3_prof_collect(phases, 9, nullptr);
  if (st != MMH3_OK) return st;
  for (int i = 0; i < n_kernels && i < MMH3_PROF_KERNELS; ++i) {
    ms[i] = g_prof_kms[i];
    if (calls) calls[i] = g_prof_kcalls[i];
  }
  return MMH3_OK;
}

void mmh3_prof_reset(void) {
  for (double& v : g_prof_ms) v = 0.0;
  for (double& v : g_prof_kms) v = 0.0;
  for (long& v : g_prof_kcalls) v = 0;
  g_prof_blocks = 0;
}

}  // extern "C"
