// Host-side planning: the packed layouts, the flow-clock remap, the
// distinct-timestep list and the segment -> adaLN row table, plus the
// library's error reporting and host fault injection.
//
// Follows "cortiq_engine/mmh3.rs" (cortiq-engine 0.5.72): the
// flow-schedule remap (time_shift_sigma), the packed layout
// (axis_from_sqrt_area, push_audio_grid, Layout::build_full) and the
// timestep / row assembly at the top of MiniMaxH3::forward.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <vector>

#include "mmh3_internal.h"

namespace mmh3 {

static std::atomic<long long> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// ------------------------------------------------------------------ errors
static thread_local char g_msg[512] = "";

mmh3_status fail(mmh3_status code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return code;
}

void clear_error() { g_msg[0] = 0; }

bool fault_injected(const char* site) {
  const char* f = std::getenv("MMH3_FAULT");
  return f != nullptr && std::strcmp(f, site) == 0;
}

mmh3_status cuda_fail(cudaError_t e, const char* what) {
  return fail(MMH3_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

static int g_check_override = -1;  // mmh3_set_check; -1: the environment decides

bool check_mode() {
  if (g_check_override >= 0) return g_check_override != 0;
  static const bool env_on = [] {
    const char* v = std::getenv("MMH3_CHECK");
    return v != nullptr && std::atoi(v) != 0;
  }();
  return env_on;
}

static uint64_t g_limit_override = 0;

uint64_t wait_limit_ns() {
  if (g_limit_override) return g_limit_override;
  static uint64_t env_limit = [] {
    const char* s = std::getenv("MMH3_WAIT_LIMIT_MS");
    double ms = s ? std::atof(s) : 2000.0;
    if (!(ms > 0)) ms = 2000.0;
    return (uint64_t)(ms * 1e6);
  }();
  return env_limit;
}

// ------------------------------------------------------------------- plan
// Where condition rows sit on the schedule ("cortiq_engine/mmh3.rs",
// VISUAL_COND_TIMESTEP and AUDIO_COND_TIMESTEP, the model's cond_aug and
// cond_aug_audio): a keyframe or reference row is all but arrived.
constexpr double kVisualCondTimestep = 0.999;
constexpr double kAudioCondTimestep = 1.0;

void curve_coords(double t, int grid, int* i0, float* f) {
  const double tc = t < 0.0 ? 0.0 : (t > 1.0 ? 1.0 : t);
  const double p = tc * (double)(grid - 1);
  int i = (int)std::floor(p);
  if (i > grid - 2) i = grid - 2;
  *i0 = i;
  *f = (float)(p - (double)i);
}

mmh3_status make_plan(const mmh3_segment* segs, int n_seg, int n, double sigma_v, double sigma_a,
                      Plan* p) {
  if (fault_injected("plan")) return fail(MMH3_ERR_ARG, "injected fault at plan");
  if (segs == nullptr || p == nullptr) return fail(MMH3_ERR_ARG, "null segment table");
  if (n_seg < 1 || n_seg > kMaxSeg) return fail(MMH3_ERR_SHAPE, "n_seg=%d not in [1, %d]", n_seg, kMaxSeg);
  if (n < 1) return fail(MMH3_ERR_SHAPE, "n=%d < 1", n);
  uint32_t expect = 0;
  bool used[kClocks] = {false, false, false, false};
  for (int k = 0; k < n_seg; ++k) {
    const mmh3_segment& s = segs[k];
    if (s.start != expect || s.stop <= s.start)
      return fail(MMH3_ERR_SHAPE, "segment %d [%u, %u) is not contiguous from %u", k, s.start, s.stop, expect);
    if (s.tag > 2) return fail(MMH3_ERR_ARG, "segment %d: tag %d not in {0,1,2}", k, (int)s.tag);
    if (s.clock >= kClocks) return fail(MMH3_ERR_ARG, "segment %d: clock %d not in [0, 3]", k, (int)s.clock);
    used[s.clock] = true;
    expect = s.stop;
  }
  if ((int)expect != n) return fail(MMH3_ERR_SHAPE, "segments cover [0, %u), n = %d", expect, n);
  // forward(): sigma_v clamped at 1e-6; t_v = 1 - sigma_v, t_a = 1 - sigma_a;
  // condition rows sit at t_cond = max(t_v, 0.999) (visual) and
  // t_cond_a = max(t_a, 1) (audio), the model's VISUAL_COND_TIMESTEP and
  // AUDIO_COND_TIMESTEP; the distinct timesteps of the clocks the segments
  // use, sorted ascending; a clock's slot is its index in that list.
  const double sv = sigma_v > 1e-6 ? sigma_v : 1e-6;
  const double t_v = 1.0 - sv, t_a = 1.0 - sigma_a;
  const double t_of[kClocks] = {t_v, t_a, std::max(t_v, kVisualCondTimestep), std::max(t_a, kAudioCondTimestep)};
  std::vector<double> ts;
  for (int c = 0; c < kClocks; ++c)
    if (used[c]) ts.push_back(t_of[c]);
  std::sort(ts.begin(), ts.end());
  ts.erase(std::unique(ts.begin(), ts.end()), ts.end());
  *p = Plan{};
  p->n_ts = (int)ts.size();
  for (size_t i = 0; i < ts.size(); ++i) p->ts[i] = ts[i];
  for (int c = 0; c < kClocks; ++c) {
    p->slot[c] = -1;
    if (!used[c]) continue;
    for (int i = 0; i < p->n_ts; ++i)
      if (p->ts[i] == t_of[c]) p->slot[c] = i;
  }
  p->block_rows.n = p->final_rows.n = n_seg;
  if (check_mode()) {  // rows outside the modulation buffer are recorded on the device
    p->block_rows.limit = 3 * p->n_ts;
    p->final_rows.limit = p->n_ts;
    p->block_rows.status = p->final_rows.status = device_status_ptr();
  }
  for (int k = 0; k < n_seg; ++k) {
    const int slot = p->slot[segs[k].clock];
    p->block_rows.start[k] = p->final_rows.start[k] = (int)segs[k].start;
    p->block_rows.stop[k] = p->final_rows.stop[k] = (int)segs[k].stop;
    p->block_rows.row[k] = slot * 3 + segs[k].tag;
    p->final_rows.row[k] = slot;
    p->seg_tag[k] = segs[k].tag;
  }
  return MMH3_OK;
}

}  // namespace mmh3

using namespace mmh3;

// ------------------------------------------------------------ public helpers
extern "C" {

double mmh3_time_shift_sigma(double sigma, double from_shift, double to_shift) {
  const double base = sigma / (from_shift + sigma * (1.0 - from_shift));
  return to_shift * base / (1.0 + (to_shift - 1.0) * base);
}

const char* mmh3_last_error(void) { return g_msg; }

const char* mmh3_version(void) { return "mmh3-b200 0.1 (sm_100a)"; }

void mmh3_set_wait_limit_ns(uint64_t ns) { g_limit_override = ns; }

void mmh3_set_check(int on) {
  g_check_override = on < 0 ? -1 : (on != 0 ? 1 : 0);
  device_status_ptr();  // writes the flag on the current device (if there is one)
}

int mmh3_check_enabled(void) { return check_mode() ? 1 : 0; }

}  // extern "C"

namespace {

// Patch-centre coordinates along one axis: n = dim/patch entries
// (i * ratio / n + (1 - ratio) / 2) * 32 with ratio = dim / sqrt_area.
std::vector<double> axis_from_sqrt_area(int dim, int patch, double sqrt_area) {
  const double ratio = (double)dim / sqrt_area;
  const int n = dim / patch;
  std::vector<double> v(n);
  for (int i = 0; i < n; ++i) v[i] = ((double)i * (ratio / (double)n) + (1.0 - ratio) / 2.0) * 32.0;
  return v;
}

struct LayoutBuilder {
  std::vector<double> pos;  // 3 per row
  std::vector<mmh3_segment> segs;
  void row(double t, double h, double w) {
    pos.push_back(t);
    pos.push_back(h);
    pos.push_back(w);
  }
  int rows() const { return (int)(pos.size() / 3); }
  void seg(int start, int tag, int clock) {
    mmh3_segment s{};
    s.start = (uint32_t)start;
    s.stop = (uint32_t)rows();
    s.tag = (uint8_t)tag;
    s.clock = (uint8_t)clock;
    segs.push_back(s);
  }
  mmh3_status emit(mmh3_segment* out_segs, int seg_cap, int* n_seg, float* out_pos, int cap, int* n_out) {
    if (n_seg == nullptr || n_out == nullptr || out_segs == nullptr)
      return fail(MMH3_ERR_ARG, "layout: null output pointer");
    *n_out = rows();
    *n_seg = (int)segs.size();
    if ((int)segs.size() > kMaxSeg)
      return fail(MMH3_ERR_SHAPE, "layout: %d segments, above the %d a block takes", (int)segs.size(), kMaxSeg);
    if ((int)segs.size() > seg_cap)
      return fail(MMH3_ERR_SHAPE, "layout: segment capacity %d < %d segments", seg_cap, (int)segs.size());
    for (size_t k = 0; k < segs.size(); ++k) out_segs[k] = segs[k];
    if (out_pos == nullptr) return MMH3_OK;
    if (cap < rows()) return fail(MMH3_ERR_SHAPE, "layout: pos capacity %d < %d rows", cap, rows());
    for (size_t i = 0; i < pos.size(); ++i) out_pos[i] = (float)pos[i];
    return MMH3_OK;
  }
};


// The packed layout of "cortiq_engine/mmh3.rs" Layout::build_full: the
// text rows (i, 0, 0) in runs of equal modality tag (text_tags, or all
// text); the reference blocks in order, each advancing the cursor (a still:
// its own h/w grid at the cursor, +1; standalone audio: t stereo frames,
// +t; a clip: its soundtrack first, then its frames stepping t by the
// 5/3 x [1,4,4,4,4] spans, + max(audio frames, spans)); the keyframes on the
// target grid, pinned to the frame they stand for without moving the
// cursor (the first frame at the cursor, the last one at cursor + spans -
// 5/3); then the target audio and the target video from the cursor.
// Segment clocks: text, audio and video on the flow clocks 0 / 1 / 0,
// keyframes and reference frames tag video on clock 2, reference audio tag
// audio on clock 3 (MiniMaxH3::forward's row assignment).
mmh3_status build_layout(LayoutBuilder& L, int text_len, int latent_t, int lat_h, int lat_w, int audio_t,
                         const mmh3_keyframe* frames, int n_frames, const mmh3_ref* refs, int n_refs,
                         const uint8_t* text_tags) {
  if (text_len < 1 || latent_t < 1 || lat_h < 2 || lat_w < 2 || audio_t < 1 || (lat_h & 1) || (lat_w & 1))
    return fail(MMH3_ERR_SHAPE, "layout: bad sizes text=%d t=%d h=%d w=%d audio=%d", text_len, latent_t, lat_h,
                lat_w, audio_t);
  if (n_frames < 0 || (n_frames > 0 && frames == nullptr) || n_refs < 0 || (n_refs > 0 && refs == nullptr))
    return fail(MMH3_ERR_ARG, "layout: keyframe / reference list null or negative");
  static const double kFramePerToken[5] = {1.0, 4.0, 4.0, 4.0, 4.0};
  const double kRescale = 5.0 / 3.0;
  const double area = std::sqrt((double)lat_h * (double)lat_w);
  const std::vector<double> hs = axis_from_sqrt_area(lat_h, 2, area);
  const std::vector<double> ws = axis_from_sqrt_area(lat_w, 2, area);
  auto audio_grid = [&](double cursor, int t, double w_low, double w_high) {
    for (int ch = 0; ch < 2; ++ch)
      for (int i = 0; i < t; ++i) L.row(cursor + (double)i, 0.0, ch == 0 ? w_low : w_high);
  };
  // text, in runs of one tag
  int run0 = 0, prev = -1;
  for (int i = 0; i < text_len; ++i) {
    const int tag = text_tags ? text_tags[i] : 1;
    if (tag > 2) return fail(MMH3_ERR_ARG, "layout: text tag %d of token %d not in {0,1,2}", tag, i);
    if (i > 0 && tag != prev) {
      L.seg(run0, prev, 0);
      run0 = L.rows();
    }
    L.row((double)i, 0.0, 0.0);
    prev = tag;
  }
  L.seg(run0, prev, 0);
  double cursor = (double)text_len;
  for (int r = 0; r < n_refs; ++r) {
    const mmh3_ref& ref = refs[r];
    if (ref.kind == MMH3_REF_IMAGE) {
      if (ref.lat_h < 2 || ref.lat_w < 2 || (ref.lat_h & 1) || (ref.lat_w & 1))
        return fail(MMH3_ERR_SHAPE, "layout: reference image %d grid %d x %d", r, ref.lat_h, ref.lat_w);
      const double a = std::sqrt((double)ref.lat_h * (double)ref.lat_w);
      const std::vector<double> rh = axis_from_sqrt_area(ref.lat_h, 2, a), rw = axis_from_sqrt_area(ref.lat_w, 2, a);
      const int s0 = L.rows();
      for (double h : rh)
        for (double w : rw) L.row(cursor, h, w);
      L.seg(s0, 0, 2);
      cursor += 1.0;
    } else if (ref.kind == MMH3_REF_AUDIO) {
      if (ref.audio_t < 0) return fail(MMH3_ERR_SHAPE, "layout: reference audio %d frames %d", r, ref.audio_t);
      if (ref.audio_t > 0) {
        const int s0 = L.rows();
        audio_grid(cursor, ref.audio_t, ws.front(), ws.back());
        L.seg(s0, 2, 3);
      }
      cursor += (double)ref.audio_t;
    } else if (ref.kind == MMH3_REF_VIDEO) {
      if (ref.latent_t < 1 || ref.audio_t < 0 || ref.lat_h < 2 || ref.lat_w < 2 || (ref.lat_h & 1) ||
          (ref.lat_w & 1))
        return fail(MMH3_ERR_SHAPE, "layout: reference clip %d sizes", r);
      const double a = std::sqrt((double)ref.lat_h * (double)ref.lat_w);
      const std::vector<double> rh = axis_from_sqrt_area(ref.lat_h, 2, a), rw = axis_from_sqrt_area(ref.lat_w, 2, a);
      if (ref.audio_t > 0) {
        const int s0 = L.rows();
        audio_grid(cursor, ref.audio_t, rw.front(), rw.back());
        L.seg(s0, 2, 3);
      }
      const int s0 = L.rows();
      double t = cursor;
      for (int k = 0; k < ref.latent_t; ++k) {
        for (double h : rh)
          for (double w : rw) L.row(t, h, w);
        t += kRescale * kFramePerToken[k % 5];
      }
      L.seg(s0, 0, 2);
      double spans = 0.0;
      for (int k = 0; k < ref.latent_t; ++k) spans += kRescale * kFramePerToken[k % 5];
      cursor += std::max((double)ref.audio_t, spans);
    } else {
      return fail(MMH3_ERR_ARG, "layout: reference %d kind %d not in {0,1,2}", r, ref.kind);
    }
  }
  // keyframes: on the target grid, never moving the cursor
  double spans = 0.0;
  for (int k = 0; k < latent_t; ++k) spans += kRescale * kFramePerToken[k % 5];
  for (int f = 0; f < n_frames; ++f) {
    const mmh3_keyframe& kf = frames[f];
    double cond_t;
    if (kf.pixel_index == 0)
      cond_t = cursor;
    else if (kf.frame_count > 0 && kf.pixel_index == kf.frame_count - 1)
      cond_t = cursor + spans - kRescale;
    else
      return fail(MMH3_ERR_ARG, "layout: keyframe %d at pixel %d of %d: only the first and last frame anchor one", f,
                  kf.pixel_index, kf.frame_count);
    const int s0 = L.rows();
    for (double h : hs)
      for (double w : ws) L.row(cond_t, h, w);
    L.seg(s0, 0, 2);
  }
  // stereo audio, channel-major, w pinned to the target grid's extremes
  const int a0 = L.rows();
  audio_grid(cursor, audio_t, ws.front(), ws.back());
  L.seg(a0, /*tag audio*/ 2, /*clock*/ 1);
  // video: t advances by the per-token frame spans
  const int v0 = L.rows();
  double t = cursor;
  for (int k = 0; k < latent_t; ++k) {
    for (double h : hs)
      for (double w : ws) L.row(t, h, w);
    t += kRescale * kFramePerToken[k % 5];
  }
  L.seg(v0, /*tag video*/ 0, /*clock*/ 0);
  return MMH3_OK;
}

}  // namespace

extern "C" mmh3_status mmh3_layout_t2va(int text_len, int latent_t, int lat_h, int lat_w,
                                        int audio_t, mmh3_segment* segs, int* n_seg, float* pos,
                                        int pos_capacity, int* n_out) {
  clear_error();
  LayoutBuilder L;
  mmh3_status st = build_layout(L, text_len, latent_t, lat_h, lat_w, audio_t, nullptr, 0, nullptr, 0, nullptr);
  if (st != MMH3_OK) return st;
  return L.emit(segs, 3, n_seg, pos, pos_capacity, n_out);
}

extern "C" mmh3_status mmh3_layout_fl2va(int text_len, int latent_t, int lat_h, int lat_w, int audio_t,
                                         const mmh3_keyframe* frames, int n_frames, const uint8_t* text_tags,
                                         mmh3_segment* segs, int seg_capacity, int* n_seg, float* pos,
                                         int pos_capacity, int* n_out) {
  clear_error();
  LayoutBuilder L;
  mmh3_status st =
      build_layout(L, text_len, latent_t, lat_h, lat_w, audio_t, frames, n_frames, nullptr, 0, text_tags);
  if (st != MMH3_OK) return st;
  return L.emit(segs, seg_capacity, n_seg, pos, pos_capacity, n_out);
}

extern "C" mmh3_status mmh3_layout_ref2va(int text_len, int latent_t, int lat_h, int lat_w, int audio_t,
                                          const mmh3_ref* refs, int n_refs, const uint8_t* text_tags,
                                          mmh3_segment* segs, int seg_capacity, int* n_seg, float* pos,
                                          int pos_capacity, int* n_out) {
  clear_error();
  LayoutBuilder L;
  mmh3_status st = build_layout(L, text_len, latent_t, lat_h, lat_w, audio_t, nullptr, 0, refs, n_refs, text_tags);
  if (st != MMH3_OK) return st;
  return L.emit(segs, seg_capacity, n_seg, pos, pos_capacity, n_out);
}

extern "C" mmh3_status mmh3_layout_image(int text_len, int ref_lat_h, int ref_lat_w, int lat_h,
                                         int lat_w, mmh3_segment* segs, int* n_seg, float* pos,
                                         int pos_capacity, int* n_out) {
  clear_error();
  if (text_len < 1 || ref_lat_h < 2 || ref_lat_w < 2 || lat_h < 2 || lat_w < 2)
    return fail(MMH3_ERR_SHAPE, "image layout: bad sizes");
  LayoutBuilder L;
  for (int i = 0; i < text_len; ++i) L.row((double)i, 0.0, 0.0);
  L.seg(0, 1, 0);
  double cursor = (double)text_len;
  const int grids[2][2] = {{ref_lat_h, ref_lat_w}, {lat_h, lat_w}};
  for (int g = 0; g < 2; ++g) {
    const int lh = grids[g][0], lw = grids[g][1];
    const double area = std::sqrt((double)lh * (double)lw);
    const std::vector<double> hs = axis_from_sqrt_area(lh, 2, area);
    const std::vector<double> ws = axis_from_sqrt_area(lw, 2, area);
    int s0 = L.rows();
    for (double h : hs)
      for (double w : ws) L.row(cursor, h, w);
    L.seg(s0, 0, 0);
    cursor += 1.0;
  }
  return L.emit(segs, 3, n_seg, pos, pos_capacity, n_out);
}

extern "C" mmh3_status mmh3_plan_timesteps(const mmh3_segment* segs, int n_seg, int n,
                                           double sigma_v, double sigma_a, double* ts, int* n_ts,
                                           int* seg_rows) {
  clear_error();
  if (ts == nullptr || n_ts == nullptr || seg_rows == nullptr)
    return fail(MMH3_ERR_ARG, "plan_timesteps: null output pointer");
  Plan p;
  mmh3_status st = make_plan(segs, n_seg, n, sigma_v, sigma_a, &p);
  if (st != MMH3_OK) return st;
  *n_ts = p.n_ts;
  for (int i = 0; i < p.n_ts; ++i) ts[i] = p.ts[i];
  for (int k = 0; k < n_seg; ++k) seg_rows[k] = p.block_rows.row[k];
  return MMH3_OK;
}

extern "C" long long mmh3_launch_count(void) { return mmh3::g_launches.load(std::memory_order_relaxed); }
