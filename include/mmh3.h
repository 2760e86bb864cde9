/*
 * mmh3.h -- C ABI of the B200 (sm_100a) packed multimodal DiT block library.
 *
 * The hot path is the forward pass of a MiniMax-H3-shaped packed-token DiT
 * block: one sequence [text | audio | video] with no batching and no
 * cross-attention, modulated per token through a segment table over a
 * rank-24 adaLN timestep curve.  Operations follow the page
 * "cortiq_engine/mmh3.rs" (docs.rs, cortiq-engine 0.5.72); the encoder-layer
 * entry points follow "ffai-argus 0.7.0 src/siglip.rs".
 *
 * Conventions (every entry point):
 *  - Matrices are row-major; projection weights are [out, in].
 *  - "device" pointers are CUDA device memory owned by the caller; "host"
 *    pointers are ordinary host memory.  The library never allocates or
 *    frees device memory and never synchronises the stream, except where an
 *    entry point says so (mmh3_device_status).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy stream).
 *  - Argument errors are reported before anything is launched; the return
 *    value is an mmh3_status and mmh3_last_error() gives a message (thread
 *    local, valid until the next call on the same thread).
 *  - Activation / GEMM-operand dtype: MMH3_BF16 (bf16 storage, fp32
 *    accumulate on tcgen05 kind::f16) or MMH3_F32 (fp32 storage, tcgen05
 *    kind::tf32).  The residual stream x is always fp32.  Norm gains, adaLN
 *    basis / bias / table and output-head biases are always fp32.
 *  - Kernel waits are bounded (default 2 s, MMH3_WAIT_LIMIT_MS or
 *    mmh3_set_wait_limit_ns); a kernel that gives up records a device status
 *    that mmh3_device_status() returns as MMH3_ERR_TIMEOUT.
 *  - The block's kernels use programmatic dependent launch: each is launched
 *    with programmatic stream serialization, lets the next kernel of the
 *    stream launch early, and waits (griddepcontrol.wait) for its
 *    predecessor before touching global memory.  A caller's own kernel
 *    launched after them without that attribute runs in plain stream order;
 *    one launched with it must itself wait before reading their outputs.
 *  - Stream capture: the forward entry points (block, stack, encoder layer,
 *    attention, token refiner, the whole denoise call) put only kernel
 *    launches, asynchronous copies and memsets on `stream`, so they can be
 *    captured into a CUDA graph (the programmatic launches become
 *    programmatic edges).  Make one uncaptured call on the
 *    device first: the first call writes the check-mode flag into the status
 *    word with a synchronous copy.  mmh3_device_status, mmh3_status_sync,
 *    mmh3_prof_collect and the host-buffer pipeline's first call synchronise
 *    and are not capturable.
 */
#ifndef MMH3_H_
#define MMH3_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MMH3_OK = 0,
  MMH3_ERR_ARG = 1,          /* null pointer, bad enum, inconsistent argument */
  MMH3_ERR_SHAPE = 2,        /* unsupported or inconsistent sizes */
  MMH3_ERR_ALIGN = 3,        /* a pointer is not 16-byte aligned */
  MMH3_ERR_WORKSPACE = 4,    /* workspace missing or too small */
  MMH3_ERR_UNSUPPORTED = 5,  /* more than two distinct timesteps, etc. */
  MMH3_ERR_CUDA = 6,         /* a CUDA runtime / driver call failed */
  MMH3_ERR_TIMEOUT = 7,      /* a kernel gave up waiting (device status) */
  MMH3_ERR_CHECK = 8         /* a device check of the MMH3_CHECK mode failed (device status) */
} mmh3_status;

typedef enum { MMH3_F32 = 0, MMH3_BF16 = 1 } mmh3_dtype;

/* Block hyper-parameters.  rope_k = rotary frequencies per position axis
 * (3*rope_k pairs rotate, dims >= 6*rope_k do not); 16 for head_dim 128. */
typedef struct {
  int hidden;        /* H, multiple of 128 */
  int heads;         /* nh */
  int head_dim;      /* hd: 64 or 128; inner = heads*head_dim == hidden */
  int ffn;           /* F (SwiGLU inner), multiple of 128 */
  int rank;          /* adaLN curve rank R (24), <= 32 */
  int grid;          /* timestep-curve table rows G (1025) */
  int rope_k;        /* hd/8 */
  float eps;         /* RMSNorm eps for norm1 / norm2 / final norm (1e-5) */
  float qk_eps;      /* q/k RMSNorm eps (1e-5) */
  float rope_theta;  /* rotary base (10000) */
  int act_dtype;     /* mmh3_dtype of activations and projection weights */
} mmh3_dims;

/* One contiguous run of tokens sharing a modality tag and a clock.
 * tag: 0 video, 1 text, 2 audio (adaLN row order).  clock: 0 = the video
 * clock (t_v = 1 - max(sigma_v, 1e-6)), 1 = the audio clock
 * (t_a = 1 - sigma_a), 2 = the visual condition clock (keyframe and
 * reference-image rows: max(t_v, 0.999)), 3 = the audio condition clock
 * (reference audio rows: max(t_a, 1)) ("cortiq_engine/mmh3.rs", forward:
 * VISUAL_COND_TIMESTEP, AUDIO_COND_TIMESTEP).  Text uses the video clock.
 * Segments must be sorted, contiguous and cover [0, n) exactly; at most
 * 16.  A token's adaLN row is slot*3 + tag, slot the index of its clock's
 * timestep among the distinct timesteps of the clocks in use (ascending).
 * The block's own adaLN basis holds two slots: more than two distinct
 * timesteps need the caller's modulation (mmh3_block_forward's
 * mods_or_null); every other entry point then returns
 * MMH3_ERR_UNSUPPORTED. */
typedef struct {
  uint32_t start, stop;
  uint8_t tag, clock;
  uint8_t pad[2];
} mmh3_segment;

/* One block's weights (device pointers).
 *  norm1, norm2 [H] fp32; q_norm, k_norm [hd] fp32;
 *  wqkv [3*inner, H] act dtype, rows [q | k | v], heads contiguous;
 *  wout [H, inner]; wfc2 [H, F];
 *  wfc1 [2F, H] act dtype in the INTERLEAVED order written by
 *       mmh3_prepare_fc1 (not the checkpoint's [gate | up] order);
 *  adaln_w [2*3*6*H, R], adaln_b [2*3*6*H], adaln_table [G, R] fp32. */
typedef struct {
  const float* norm1;
  const float* norm2;
  const void* wqkv;
  const void* wout;
  const float* q_norm;
  const float* k_norm;
  const void* wfc1;
  const void* wfc2;
  const float* adaln_w;
  const float* adaln_b;
  const float* adaln_table;
} mmh3_block_weights;

/* Final layer (output heads).  final_norm [H] fp32; adaln_w [2*2*H, R],
 * adaln_b [2*2*H], adaln_table [G, R] fp32 (one modality, chunks shift,
 * scale); w_video [out_video, H] / w_audio [out_audio, H] act dtype;
 * b_video / b_audio fp32.  out_* must be multiples of 32. */
typedef struct {
  const float* final_norm;
  const float* adaln_w;
  const float* adaln_b;
  const float* adaln_table;
  const void* w_video;
  const float* b_video;
  const void* w_audio;
  const float* b_audio;
  int out_video;
  int out_audio;
} mmh3_head_weights;

/* ------------------------------------------------------------ host helpers */

/* sigma on the to_shift schedule at the same base-grid point:
 * b = s / (f + s (1 - f)),  s' = t b / (1 + (t - 1) b)
 * ("cortiq_engine/mmh3.rs", time_shift_sigma).  Host only, never fails. */
double mmh3_time_shift_sigma(double sigma, double from_shift, double to_shift);

/* The t2va layout [text | audio | video] ("cortiq_engine/mmh3.rs",
 * Layout::t2va / build_full): text rows (i, 0, 0); stereo audio rows
 * channel-major from t = text_len with w at the frame grid's extremes; video
 * frames advancing t by (5/3)*[1,4,4,4,4][k%5] over the 2x2-patch h/w grid
 * of axis_from_sqrt_area.  Positions are computed in fp64 and rounded to
 * fp32.  Host buffers: segs [>= 3], pos [pos_capacity * 3] (t, h, w).
 * *n_out = text_len + 2*audio_t + latent_t*(lat_h/2)*(lat_w/2); returns
 * MMH3_ERR_SHAPE if pos_capacity is smaller (pos may be NULL to query n). */
mmh3_status mmh3_layout_t2va(int text_len, int latent_t, int lat_h, int lat_w, int audio_t,
                             mmh3_segment* segs, int* n_seg, float* pos, int pos_capacity,
                             int* n_out);

/* A keyframe of fl2va: the pixel frame it stands for and the clip's frame
 * count.  Only the first (pixel_index 0) and the last (frame_count - 1)
 * frame can anchor one. */
typedef struct {
  int pixel_index, frame_count;
} mmh3_keyframe;

/* A reference block of ref2va, in the order given.
 *  MMH3_REF_IMAGE: a still of lat_h x lat_w latents (even);
 *  MMH3_REF_AUDIO: audio_t standalone audio frames (stereo);
 *  MMH3_REF_VIDEO: latent_t frames of lat_h x lat_w latents with an
 *                  optional soundtrack of audio_t frames packed before
 *                  them from the same origin. */
#define MMH3_REF_IMAGE 0
#define MMH3_REF_AUDIO 1
#define MMH3_REF_VIDEO 2
typedef struct {
  int kind;
  int lat_h, lat_w;
  int latent_t;
  int audio_t;
} mmh3_ref;

/* fl2va ("cortiq_engine/mmh3.rs", Layout::fl2va / build_full):
 * [text | keyframes | audio | video].  Keyframe rows take the target's
 * 2x2-patch grid at the time of the frame they stand for -- the first frame
 * at the text's end, the last one at text_len + spans - 5/3 (spans = the
 * target's summed 5/3 x [1,4,4,4,4] frame spans) -- and never move the
 * cursor, so the audio and the video start where t2va puts them.  Keyframe
 * segments are tag video on clock 2.  text_tags (host, text_len entries, or
 * NULL = all text) gives each prompt token's modality tag; runs of one tag
 * become separate text segments on clock 0.  Host buffers: segs
 * [seg_capacity], pos [pos_capacity * 3] (pos may be NULL to query n).
 * MMH3_ERR_ARG for a keyframe that is neither the first nor the last
 * frame; MMH3_ERR_SHAPE if the segments exceed seg_capacity or 16. */
mmh3_status mmh3_layout_fl2va(int text_len, int latent_t, int lat_h, int lat_w, int audio_t,
                              const mmh3_keyframe* frames, int n_frames, const uint8_t* text_tags,
                              mmh3_segment* segs, int seg_capacity, int* n_seg, float* pos,
                              int pos_capacity, int* n_out);

/* ref2va ("cortiq_engine/mmh3.rs", Layout::ref2va / build_full):
 * [text | references | audio | video].  Each reference advances the cursor:
 * a still puts its own h/w grid at the cursor, +1; standalone audio its
 * stereo frames from the cursor, +audio_t; a clip its soundtrack (w at its
 * own grid's extremes) and then its frames (t stepping by the frame
 * spans), + max(audio_t, spans).  The target audio and video start at the
 * final cursor.  Reference frames are tag video on clock 2, reference audio
 * tag audio on clock 3.  Buffers and errors as mmh3_layout_fl2va. */
mmh3_status mmh3_layout_ref2va(int text_len, int latent_t, int lat_h, int lat_w, int audio_t,
                               const mmh3_ref* refs, int n_refs, const uint8_t* text_tags,
                               mmh3_segment* segs, int seg_capacity, int* n_seg, float* pos,
                               int pos_capacity, int* n_out);

/* Image mode [text | reference image | target image]: the reference image is
 * placed like a reference still of "cortiq_engine/mmh3.rs" build_full (rows
 * at the cursor t with their own h/w grid, cursor + 1), the target at the
 * next t; image rows are tag video on clock 0.  Same buffers as above. */
mmh3_status mmh3_layout_image(int text_len, int ref_lat_h, int ref_lat_w, int lat_h, int lat_w,
                              mmh3_segment* segs, int* n_seg, float* pos, int pos_capacity,
                              int* n_out);

/* Distinct timesteps (ascending, de-duplicated) of the clocks the segments
 * use, and each segment's block adaLN row slot(clock)*3 + tag
 * ("cortiq_engine/mmh3.rs", forward).  Host buffers: ts [4], seg_rows
 * [n_seg].  Up to four timesteps (the four clocks). */
mmh3_status mmh3_plan_timesteps(const mmh3_segment* segs, int n_seg, int n, double sigma_v,
                                double sigma_a, double* ts, int* n_ts, int* seg_rows);

/* ------------------------------------------------------------ device steps */

/* Writes the per-token adaLN row (int32 [n], device) that the fused
 * norm/modulate gather uses: rows[i] = slot(clock)*3 + tag of i's segment. */
mmh3_status mmh3_resolve_rows(const mmh3_segment* segs, int n_seg, int n, double sigma_v,
                              double sigma_a, int32_t* rows_dev, void* stream);

/* adaLN as a curve ("cortiq_engine/mmh3.rs", Adaln::eval): for each distinct
 * timestep slot s (ts from the segments, sigma_v, sigma_a):
 *   p = clamp(t,0,1)*(G-1), i0 = min(floor p, G-2), f = p - i0,
 *   c = (1-f) table[i0] + f table[i0+1],
 *   out[s*rows_per_slot + r] = w[s*rows_per_slot + r] . c + b[...]
 * rows_per_slot = 18*H for a block (3 tags x 6 chunks), 2*H for the final
 * layer.  out: device fp32 [n_ts * rows_per_slot].  *n_ts receives T_s. */
mmh3_status mmh3_adaln_modulation(const mmh3_dims* dims, const float* w, const float* b,
                                  const float* table, int rows_per_slot, const mmh3_segment* segs,
                                  int n_seg, int n, double sigma_v, double sigma_a, float* out,
                                  int* n_ts, void* stream);

/* Rewrites fc1 [2F, H] from the checkpoint order [gate | up] into the tile
 * order the fused fc1+SwiGLU kernel reads: blocks of 256 rows, 128 gate rows
 * then the 128 matching up rows ("cortiq_engine/mmh3.rs", ffn_tail: fc1's
 * output is [gate | up]).  Device in/out, act dtype, distinct buffers
 * (MMH3_ERR_ARG if null or equal, MMH3_ERR_ALIGN unless 16-byte aligned).
 * The one preparation a block's weights need; run it once per block. */
mmh3_status mmh3_prepare_block_weights(const mmh3_dims* dims, const void* fc1_gate_up,
                                       void* fc1_interleaved, void* stream);

/* The same call under its older name. */
mmh3_status mmh3_prepare_fc1(const mmh3_dims* dims, const void* fc1_gate_up, void* fc1_tiled,
                             void* stream);

/* Bytes of device workspace mmh3_block_forward / mmh3_stack_forward need for
 * n tokens.  Layout (each region 256-byte aligned, in this order): mods fp32
 * [2*3, 6H]; rope (cos, sin) fp32x2 [n, 3*rope_k]; xn1 [n, H]; qkv [n, 3*inner]
 * (q and k after qk-norm + rotation); attn [n, inner]; xn2 [n, H]; act [n, F];
 * head scratch [n, H]; final mods fp32 [2, 2H]; attention's work counter
 * (16 bytes, zeroed by the block's first RMSNorm launch) -- all act dtype
 * unless stated.  After a block call the regions hold that block's
 * intermediates. */
mmh3_status mmh3_workspace_size(const mmh3_dims* dims, int n, size_t* bytes);

/* Full bidirectional attention over packed sequences (work units of two
 * 128-row query tiles of one head, tcgen05): for each sequence b < n_seq of `seq` tokens
 * starting at row b*seq of the qkv panel [n_seq*seq, 3*heads*head_dim]
 * (rows [q | k | v], heads contiguous, act dtype, device), per head:
 * out = softmax(q k^T * scale) v, written to out [n_seq*seq, heads*head_dim]
 * ("cortiq_engine/mmh3.rs", attention; softmax_inplace).  scale is applied
 * to the scores (pass 1/sqrt(hd); 1 when it is folded into q). */
mmh3_status mmh3_attention(const void* qkv, int n_seq, int seq, int heads, int head_dim,
                           int act_dtype, float scale, void* out, void* stream);

/* mmh3_attention with a scratch region (bf16 only).  Its first 256 bytes
 * hold a work counter (zeroed on the stream by a memset), and the launch is
 * persistent: one CTA per SM takes work items from the counter until none
 * is left.  Work units of 256 query rows of one head fill the SMs in
 * waves.  The units of the last, partial wave are split along the keys
 * into f items when that shortens the wave enough: f in 2..8 minimises
 * ceil(tail * f / SMs) / f, each piece keeps at least 32 key tiles of 128,
 * and the split is made only if the tail's time drops to 0.6 of a unit or
 * less.  The pieces come after the whole units, so the SMs that finish
 * first take them.  Their partial results (unnormalised O, running
 * maximum, row sum: 256 x (head_dim + 4) fp32 per piece) go to scratch
 * after the counter and are then merged.  With scratch NULL (or under 256
 * bytes) every item is its own CTA; without room for the partial results
 * nothing is split.  The result equals mmh3_attention's up to the order of
 * the softmax sums.  The block entry points give attention this region from
 * their workspace (the SwiGLU activation region, free until fc1; the
 * encoder layer its LayerNorm output, free between qkv and LN2). */
mmh3_status mmh3_attention_ws(const void* qkv, int n_seq, int seq, int heads, int head_dim,
                              int act_dtype, float scale, void* out, void* scratch,
                              size_t scratch_bytes, void* stream);

/* One modulated block, in place on x [n, H] fp32 (device)
 * ("cortiq_engine/mmh3.rs", block_forward + ffn_tail):
 *   mods = adaLN(ts); xn1 = RMSNorm(x; norm1)(1+scale_msa)+shift_msa;
 *   qkv = xn1 Wqkv^T; q,k = RMSNorm per head (q_norm/k_norm) + partial
 *   split-half 3-axis rotation by pos; attn = softmax(q k^T/sqrt(hd)) v;
 *   x += gate_msa * (attn Wout^T); xn2 = RMSNorm(x; norm2)(1+scale_mlp)
 *   +shift_mlp; act = silu(xn2 Wg^T) * (xn2 Wu^T); x += gate_mlp * (act W2^T).
 * The modulation row of token i is given by its segment (mmh3_segment).
 * pos_dev: device fp32 [n, 3] (t, h, w), or NULL for no rotation.
 * modulated = 0 runs the unmodulated form (plain residuals, no adaLN; the
 * weights' adaln pointers may be NULL).
 * mods_or_null: NULL evaluates the block's adaLN curve (Adaln::eval) at the
 * segments' timesteps; otherwise a device fp32 [T_s*3, 6H] modulation
 * buffer, 16-byte aligned, laid out as mmh3_adaln_modulation writes it
 * (row slot*3 + tag, chunks shift_msa, scale_msa, gate_msa, shift_mlp,
 * scale_mlp, gate_mlp), used as is: the adaLN launch is skipped and the
 * weights' adaln pointers may be NULL.  T_s and the slots still come from
 * the segments and sigmas.  Only read by the call's kernels, so it must stay
 * valid until they finish.  MMH3_ERR_ARG if given with modulated = 0.
 * workspace: mmh3_workspace_size. */
mmh3_status mmh3_block_forward(const mmh3_dims* dims, const mmh3_block_weights* w, float* x, int n,
                               const mmh3_segment* segs, int n_seg, const float* pos_dev,
                               double sigma_v, double sigma_a, int modulated,
                               const float* mods_or_null, void* workspace, size_t ws_bytes,
                               void* stream);

/* n_blocks blocks (blocks: host array of n_blocks weight structs) then,
 * if heads != NULL, the two output heads ("cortiq_engine/mmh3.rs", forward
 * "blocks" and "heads"): per stream (the video segment rows -> out_video
 * [rows, out_video], the audio segment rows -> out_audio [rows, out_audio],
 * fp32 device), RMSNorm(final_norm) -> (1+scale)+shift from the final adaLN
 * row of the stream's timestep -> W^T + b -> negated.  The rotation table is
 * computed once for all blocks. */
mmh3_status mmh3_stack_forward(const mmh3_dims* dims, const mmh3_block_weights* blocks,
                               int n_blocks, const mmh3_head_weights* heads, float* x, int n,
                               const mmh3_segment* segs, int n_seg, const float* pos_dev,
                               double sigma_v, double sigma_a, float* out_video, float* out_audio,
                               void* workspace, size_t ws_bytes, void* stream);

/* ----------------------------------------------------- block on host data */

/* Device slots of the host-buffer block (below). */
#define MMH3_HOST_SLOTS 3

/* One modulated block whose input and result live in host memory, with the
 * copies overlapped with other calls' compute.  Per call, ordered by events:
 *   copy_in_stream:  x_in_host -> x_dev and pos_host -> pos_dev (after the
 *                    previous call on the same slot has copied its result
 *                    out of x_dev);
 *   stream:          mmh3_block_forward on x_dev / pos_dev (workspace as
 *                    there);
 *   copy_out_stream: x_dev -> x_out_host.
 * The call returns at once.  Rotate the slots 0, 1, 2 (MMH3_HOST_SLOTS) with
 * one set of device buffers per slot (x_dev [n, H] fp32 and pos_dev [n, 3]
 * fp32): a call's copy-in then waits only for the copy-out of the call three
 * back, so the copy-out of call i and the copy-in of call i + 3 overlap the
 * blocks of calls i + 1 and i + 2.  With two slots the two copies would
 * have to fit within one block's time.  slot outside [0, MMH3_HOST_SLOTS)
 * returns MMH3_ERR_ARG.  Host buffers
 * must be pinned (cudaHostAlloc / cudaHostRegister) for the copies to be
 * asynchronous, and stay untouched until the call's copy-out has finished
 * (synchronize copy_out_stream).  pos_host / pos_dev may both be NULL (no
 * rotation).  The events are the library's, one set per device: calls on
 * one device must come from one host thread at a time.  No counterpart in
 * the pages; this is how a caller keeps the host transfers off the
 * critical path. */
mmh3_status mmh3_block_forward_host(const mmh3_dims* dims, const mmh3_block_weights* w,
                                    const float* x_in_host, float* x_out_host, int n,
                                    const mmh3_segment* segs, int n_seg, const float* pos_host,
                                    double sigma_v, double sigma_a, int slot, float* x_dev,
                                    float* pos_dev, void* workspace, size_t ws_bytes, void* stream,
                                    void* copy_in_stream, void* copy_out_stream);

/* ------------------------------------------- block over a sequence shard */

/* The block split at its one exchange step, for a packed sequence whose
 * rows are divided over ranks in contiguous shards (context parallelism;
 * "cortiq_engine/mmh3.rs", block_forward, with attention over the whole
 * sequence).  Each rank calls begin on its shard, the caller all-gathers
 * the K|V rows of all shards in sequence order (for example NCCL
 * all-gather on the same stream), then each rank calls end.  Shard
 * arguments: x [n, H] fp32 holds the shard's rows; segs are the shard's
 * segments with rows counted from the shard's first row (the tags and
 * clocks of the segments it intersects); pos_dev [n, 3] the shard's
 * positions.  bf16 activations only (MMH3_ERR_UNSUPPORTED otherwise).
 *
 * begin: adaLN, rotation table, norm1 + modulate, qkv GEMM with q/k norm and
 * rotation; then the shard's K|V rows (bf16, k then v, [n, 2*inner]) are
 * copied to kv_out (device, 16-byte aligned).  The workspace
 * (mmh3_workspace_size for n rows) keeps the modulation, the rotation
 * table and q for end: pass the same workspace to end, untouched. */
mmh3_status mmh3_block_cp_begin(const mmh3_dims* dims, const mmh3_block_weights* w, const float* x,
                                int n, const mmh3_segment* segs, int n_seg, const float* pos_dev,
                                double sigma_v, double sigma_a, int modulated, void* kv_out,
                                void* workspace, size_t ws_bytes, void* stream);

/* end: attention of the shard's n queries against kv_all [n_kv, 2*inner]
 * (the gathered K|V of the whole sequence, rows in sequence order; rows
 * beyond n_kv are never read), then out GEMM + gated residual, norm2 +
 * modulate, fc1 + SwiGLU, fc2 + gated residual, in place on x. */
mmh3_status mmh3_block_cp_end(const mmh3_dims* dims, const mmh3_block_weights* w, float* x, int n,
                              const mmh3_segment* segs, int n_seg, double sigma_v, double sigma_a,
                              int modulated, const void* kv_all, int n_kv, void* workspace,
                              size_t ws_bytes, void* stream);

/* --------------------------------------- token refiner, embed, unpacking */

/* Bytes of device workspace mmh3_refine_text needs for n text tokens: the
 * block workspace of mmh3_workspace_size followed (256-byte aligned) by the
 * refiner's fp32 residual stream [n, H]. */
mmh3_status mmh3_refine_workspace_size(const mmh3_dims* dims, int n, size_t* bytes);

/* The token refiner ("cortiq_engine/mmh3.rs", MiniMaxH3::refine_text):
 *   h = states cond_w^T + cond_b;
 *   each of the n_blocks refiner blocks, unmodulated and unrotated (plain
 *   residuals; q/k still get their per-head RMSNorm);
 *   out = RMSNorm(h; refiner_norm, final_eps).
 * states [n, text_dim] and cond_w [H, text_dim] act dtype, text_dim * the
 * element size a multiple of 16 bytes; cond_b and refiner_norm [H] fp32;
 * blocks: host array of n_blocks weight structs (their adaLN pointers are
 * not read and may be NULL); out [n, H] fp32.  Device pointers, 16-byte
 * aligned.  The workspace is mmh3_refine_workspace_size bytes. */
mmh3_status mmh3_refine_text(const mmh3_dims* dims, const void* states, int n, int text_dim,
                             const void* cond_w, const float* cond_b,
                             const mmh3_block_weights* blocks, int n_blocks,
                             const float* refiner_norm, float final_eps, float* out,
                             void* workspace, size_t ws_bytes, void* stream);

/* Stream kinds of mmh3_patch_embed (the segment tag of the rows written). */
#define MMH3_STREAM_VIDEO 0
#define MMH3_STREAM_AUDIO 2

/* Bytes of device workspace mmh3_patch_embed needs: the staged patch rows
 * [rows, K] in act dtype (see below for rows and K). */
mmh3_status mmh3_patch_embed_workspace_size(const mmh3_dims* dims, int kind, int channels,
                                            int frames, int lat_h, int lat_w, size_t* bytes);

/* One stream's latents -> its rows of the packed hidden states
 * ("cortiq_engine/mmh3.rs", forward "embed", patchify_video, pack_audio):
 *  kind MMH3_STREAM_VIDEO: latents [C, T, lat_h, lat_w] fp32 (lat_h, lat_w
 *    even) -> rows = T*(lat_h/2)*(lat_w/2) 2x2 patches, row (t, i, j) holding
 *    latents[c, t, 2i+p, 2j+q] at column 4c + 2p + q; K = 4C.
 *  kind MMH3_STREAM_AUDIO: latents [C, 2, T] fp32 -> rows = 2T, stereo
 *    channel 0's frames then channel 1's, row (ch, t) = latents[:, ch, t];
 *    K = C (lat_h, lat_w ignored).
 * Then x_rows[r] = rows[r] w^T + b with w [H, K] act dtype (K * element size a
 * multiple of 16 bytes) and b [H] fp32; x_rows is fp32 [rows, H], normally
 * x + start*H of the stream's segment.  The patch rows are rounded to the
 * act dtype (the projection's operand precision).  Device pointers. */
mmh3_status mmh3_patch_embed(const mmh3_dims* dims, int kind, const float* latents, int channels,
                             int frames, int lat_h, int lat_w, const void* w, const float* b,
                             float* x_rows, void* workspace, size_t ws_bytes, void* stream);

/* The inputs of one denoise evaluation's embed.  text: refined text rows
 * [>= text segment rows, H] fp32 (mmh3_refine_text); video [C_v, T_v,
 * lat_h, lat_w] and audio [C_a, 2, T_a] fp32; cond: host array of n_cond
 * device pointers, each a condition frame [C_v, 1, lat_h, lat_w] fp32 with
 * its noise blend already applied.  All device memory except `cond`. */
typedef struct {
  const float* text;
  const float* video;
  int video_channels, video_frames, lat_h, lat_w;
  const float* audio;
  int audio_channels, audio_frames;
  const float* const* cond;
  int n_cond;
} mmh3_embed_inputs;

/* The patch projections: w_video [H, 4*C_v], w_audio [H, C_a] act dtype;
 * b_video, b_audio [H] fp32 (device). */
typedef struct {
  const void* w_video;
  const float* b_video;
  const void* w_audio;
  const float* b_audio;
} mmh3_embed_weights;

/* Workspace of mmh3_embed: the largest of its mmh3_patch_embed calls. */
mmh3_status mmh3_embed_workspace_size(const mmh3_dims* dims, const mmh3_embed_inputs* in,
                                      size_t* bytes);

/* The packed hidden states x [n, H] fp32 of one denoise evaluation
 * ("cortiq_engine/mmh3.rs", forward "embed"): the first text-tag segment
 * takes the first (stop - start) text rows; the LAST video-tag segment (the
 * target) takes the video latents and the last audio-tag segment the audio
 * latents through mmh3_patch_embed; every other video-tag segment, in order,
 * takes the next condition frame through the video projection.  Each
 * segment's row count must match what its stream gives (MMH3_ERR_SHAPE
 * otherwise), and n_cond must equal the number of those other segments.
 * This places fl2va keyframes (frames on the target grid) and image-mode
 * references; reference audio (clock 3) has no input here
 * (MMH3_ERR_UNSUPPORTED), and a reference still or clip of another grid
 * fails the row-count check. */
mmh3_status mmh3_embed(const mmh3_dims* dims, const mmh3_segment* segs, int n_seg, int n,
                       const mmh3_embed_inputs* in, const mmh3_embed_weights* w, float* x,
                       void* workspace, size_t ws_bytes, void* stream);

/* The inverse of the video patchify: rows [T*(lat_h/2)*(lat_w/2), 4C] fp32
 * (the video head's output) -> out [C, T, lat_h, lat_w] fp32
 * ("cortiq_engine/mmh3.rs", unpatchify_video).  Device, distinct buffers. */
mmh3_status mmh3_unpatchify_video(const float* rows, int channels, int frames, int lat_h, int lat_w,
                                  float* out, void* stream);

/* The inverse of the audio packing: rows [2T, C] fp32 -> out [C, 2, T] fp32
 * ("cortiq_engine/mmh3.rs", unpack_audio).  Device, distinct buffers. */
mmh3_status mmh3_unpack_audio(const float* rows, int channels, int frames, float* out,
                              void* stream);

/* Bytes of device workspace mmh3_forward needs: the larger of the block
 * workspace (mmh3_workspace_size) and the embed workspace, then the video
 * head rows [T_v*(lat_h/2)*(lat_w/2), 4*C_v] and the audio head rows
 * [2*T_a, C_a], fp32, each 256-byte aligned. */
mmh3_status mmh3_forward_workspace_size(const mmh3_dims* dims, int n, const mmh3_embed_inputs* in,
                                        size_t* bytes);

/* One denoise evaluation ("cortiq_engine/mmh3.rs", MiniMaxH3::forward):
 * mmh3_embed into x [n, H] fp32, then the n_blocks blocks and both heads as
 * in mmh3_stack_forward, then the head rows unpatchified into video_out
 * [C_v, T_v, lat_h, lat_w] and unpacked into audio_out [C_a, 2, T_a] (fp32,
 * device).  The results are the two velocities, each on its own clock and
 * negated.  heads->out_video must be 4*C_v and heads->out_audio C_a
 * (MMH3_ERR_SHAPE otherwise); a stream with no segment is skipped and its
 * output pointer may be NULL.  x holds the last block's hidden states
 * afterwards. */
mmh3_status mmh3_forward(const mmh3_dims* dims, const mmh3_segment* segs, int n_seg, int n,
                         const float* pos_dev, double sigma_v, double sigma_a,
                         const mmh3_embed_inputs* in, const mmh3_embed_weights* ew,
                         const mmh3_block_weights* blocks, int n_blocks,
                         const mmh3_head_weights* heads, float* x, float* video_out,
                         float* audio_out, void* workspace, size_t ws_bytes, void* stream);

/* Size of the fixed device scratch that mmh3_block_forward_noalloc uses:
 * 32 MiB, reserved on every GPU where the library's device code is loaded,
 * until the process exits. */
#define MMH3_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/* mmh3_block_forward for callers that cannot allocate device memory (no
 * counterpart in the pages; this is a library-usage addition).  Some hosts
 * own every device allocation through their own pool and give plugins no
 * allocator, and some runtimes must not call cudaMalloc on their hot path
 * because it synchronises the device; such callers cannot provide the
 * workspace mmh3_block_forward needs.  This entry point runs the same
 * kernels with the block's intermediates in one fixed library-owned device
 * array of MMH3_NOALLOC_SCRATCH_BYTES, and allocates nothing itself: the
 * caller still passes x, the weights and the positions.
 *  - Sizes whose intermediates (mmh3_workspace_size) exceed the array are
 *    rejected with MMH3_ERR_WORKSPACE and a message giving the largest token
 *    count that fits (556 tokens at hidden 2688, 21 x 128 heads, ffn 10752).
 *  - The first call on each device looks up the array's device address with
 *    that device current; make that first call before any stream capture.
 *  - All calls share the array, which keeps the last call's contents; calls
 *    whose kernels overlap on the GPU race on it.  Nothing in it needs to
 *    start at zero.  The phase profile is not recorded by this entry point.
 *  - The cached address belongs to the CUDA context that was current at the
 *    lookup; a call made under another context on the same device (after
 *    cudaDeviceReset, for example) looks it up again.
 * Arguments and results are those of mmh3_block_forward without the
 * workspace; the modulation is always the block's own adaLN curve (no
 * mods_or_null). */
mmh3_status mmh3_block_forward_noalloc(const mmh3_dims* dims, const mmh3_block_weights* w, float* x,
                                       int n, const mmh3_segment* segs, int n_seg,
                                       const float* pos_dev, double sigma_v, double sigma_a,
                                       int modulated, void* stream);

/* ------------------------------------------------------ SigLIP encoder layer */

typedef struct {
  int hidden;     /* H, multiple of 128 */
  int heads;
  int head_dim;   /* 64 */
  int mlp;        /* multiple of 128 */
  float ln_eps;
} mmh3_vit_dims;

/* ln1_g/ln1_b/ln2_g/ln2_b [H] fp32; wqkv [3H, H] bf16 with the attention
 * scale folded into its q rows and bqkv [3H] fp32 likewise (see
 * mmh3_vit_fold_qkv); wo [H, H], w1 [mlp, H], w2 [H, mlp] bf16; bo, b1, b2
 * fp32. */
typedef struct {
  const float* ln1_g;
  const float* ln1_b;
  const void* wqkv;
  const float* bqkv;
  const void* wo;
  const float* bo;
  const float* ln2_g;
  const float* ln2_b;
  const void* w1;
  const float* b1;
  const void* w2;
  const float* b2;
} mmh3_vit_weights;

/* Fuse q/k/v into one [3H, H] bf16 matrix and [3H] fp32 bias with the
 * attention scale head_dim^-1/2 multiplied into the q rows and q bias
 * ("ffai-argus 0.7.0 src/siglip.rs", Layer::load).  Device pointers. */
mmh3_status mmh3_vit_fold_qkv(const mmh3_vit_dims* dims, const void* wq, const void* wk,
                              const void* wv, const float* bq, const float* bk, const float* bv,
                              void* wqkv, float* bqkv, void* stream);

/* Workspace: h [B*S, H] bf16, qkv [B*S, 3H] bf16, attn [B*S, H] bf16,
 * act [B*S, mlp] bf16, attention's work counter (16 bytes, zeroed by LN1)
 * (256-byte aligned regions, in this order). */
mmh3_status mmh3_vit_workspace_size(const mmh3_vit_dims* dims, int batch, int seq, size_t* bytes);

/* One pre-norm encoder layer, in place on x [batch*seq, H] fp32
 * ("ffai-argus 0.7.0 src/siglip.rs", Layer::forward + finish_attention):
 *   y = x + (attn(LN1 x) Wo^T + bo),  z = y + (gelu_tanh(LN2 y W1^T + b1) W2^T + b2)
 * with attention inside each image of `seq` tokens and LayerNorm's variance
 * computed two-pass. */
mmh3_status mmh3_vit_layer_forward(const mmh3_vit_dims* dims, const mmh3_vit_weights* w, float* x,
                                   int batch, int seq, void* workspace, size_t ws_bytes,
                                   void* stream);

/* ------------------------------------------------------------ diagnostics */

/* Synchronises `stream`, then reads and clears the device status word that
 * bounded waits write.  *code receives the first device error (0 = none);
 * returns MMH3_ERR_TIMEOUT if one was recorded. */
mmh3_status mmh3_device_status(void* stream, int* code, int* site);

/* Synchronises `stream` and reads and clears the device status word, as
 * mmh3_device_status does without the site: *device_status receives the
 * first device error code (0 = none; may be NULL); returns MMH3_ERR_TIMEOUT
 * if a kernel gave up waiting, MMH3_ERR_CUDA if the synchronisation failed.
 * The one entry point besides mmh3_device_status that waits for the GPU. */
mmh3_status mmh3_status_sync(void* stream, int* device_status);

/* The check mode (no counterpart in the pages; the memory-safety evidence
 * where no sanitizer runs).  On: MMH3_CHECK=1 in the environment, or
 * mmh3_set_check(1); mmh3_set_check(-1) returns to the environment's
 * choice.  While it is on:
 *  - every token's modulation row is checked against the modulation
 *    buffer's rows (T_s * 3 for a block, T_s for the heads), every TMA
 *    operand copy of the GEMMs and of attention against the copy rules
 *    (x offset a multiple of 16 bytes, no negative coordinate); a failure
 *    is recorded in the device status word, the access skipped (the
 *    kernel aborts through its bounded-wait path), never trapped;
 *  - each workspace region is followed by a 256-byte canary, written at the
 *    start of a call and verified after every kernel of the block, the
 *    stack and the heads (mmh3_workspace_size reports the larger size,
 *    so query it with the mode already set);
 *  - mmh3_device_status / mmh3_status_sync return MMH3_ERR_CHECK with the
 *    record (code 6 row, 7 TMA coordinate, 8 canary; the canary's site is
 *    kernel * 16 + region, kernel as MMH3_PROF_K_*, 8 for the heads).
 * The flag lives in each device's status word and is written (a
 * synchronous copy) on the first call that touches a device after the mode
 * changes: set the mode outside stream capture. */
void mmh3_set_check(int on);
int mmh3_check_enabled(void);

/* Bound on every in-kernel wait, in nanoseconds (0 restores the default). */
void mmh3_set_wait_limit_ns(uint64_t ns);

/* Launches one warp that waits on an mbarrier nothing arrives at, with a
 * wait limit of limit_ns, and synchronises the stream: exercises the
 * bounded-wait error path without hanging anything.  Returns the status
 * mmh3_device_status would (MMH3_ERR_TIMEOUT when the wait ran out). */
mmh3_status mmh3_selftest_wait_timeout(uint64_t limit_ns, void* stream);

/* Per-phase device-time profile of the block, in the nine phase slots of
 * "cortiq_engine/mmh3.rs" (MMH3_PROF): 0 norm+modulate (with the adaLN curve
 * and the rotation table), 1 qkv GEMM (qk-norm and rotation fused in; slot 2
 * stays 0), 3 attention, 4 out GEMM + gated residual, 5 fc1 GEMM + SwiGLU
 * (slot 6 stays 0), 7 fc2 GEMM + gated residual (slot 8 stays 0).
 * mmh3_prof_enable(1) makes the block entry points record CUDA events on
 * their stream between launches; mmh3_prof_collect waits for the recorded
 * events and adds their times into ms[0..min(n_slots,9)) (cumulative since
 * the last reset), with *n_blocks the number of blocks profiled.  The
 * encoder layer (mmh3_vit_layer_forward) records into the same slots and
 * counts as one block: its two LayerNorms in slot 0 (kernels NORM1, NORM2),
 * qkv + bias in 1, attention in 3, out + bias + residual in 4, fc1 + bias +
 * GELU in 5, fc2 + bias + residual in 7.  Not thread safe; the events are
 * created lazily and reused. */
void mmh3_prof_enable(int on);
mmh3_status mmh3_prof_collect(double* ms, int n_slots, long* n_blocks);
void mmh3_prof_reset(void);

/* The same intervals by kernel (a finer split of the phase slots: slot 0
 * holds the prologue and both RMSNorm + modulate launches).  The prologue
 * is one launch that evaluates the adaLN curve of one block (of up to 64
 * blocks at once in mmh3_stack_forward) and writes the rotation table.
 * Attention counts its whole step (its launch, whole units and any split
 * tail in one grid, and the merge when the tail is split). */
#define MMH3_PROF_K_PROLOGUE 0 /* adaLN curve -> modulation, rotation table */
#define MMH3_PROF_K_NORM1 1    /* segment gather + RMSNorm(norm1) + modulate */
#define MMH3_PROF_K_QKV 2      /* qkv GEMM + qk-norm + rotation */
#define MMH3_PROF_K_ATTN 3     /* attention step */
#define MMH3_PROF_K_OUT 4      /* out GEMM + gated residual */
#define MMH3_PROF_K_NORM2 5    /* segment gather + RMSNorm(norm2) + modulate */
#define MMH3_PROF_K_FC1 6      /* fc1 GEMM + SwiGLU */
#define MMH3_PROF_K_FC2 7      /* fc2 GEMM + gated residual */
#define MMH3_PROF_KERNELS 8

/* Waits for the recorded events like mmh3_prof_collect (which it calls, so
 * the phase totals are folded in too) and writes, for each kernel id below
 * n_kernels, the cumulative device time in ms[id] and, if calls is not
 * NULL, the number of timed launches in calls[id].  Reset by
 * mmh3_prof_reset. */
mmh3_status mmh3_prof_collect_kernels(double* ms, long* calls, int n_kernels);

/* Message of the last failing call on this thread ("" if none). */
const char* mmh3_last_error(void);

/* Number of kernels the library has launched in this process so far (all
 * devices, all threads).  Host only, never fails. */
long long mmh3_launch_count(void);

/* Library version string. */
const char* mmh3_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MMH3_H_ */
