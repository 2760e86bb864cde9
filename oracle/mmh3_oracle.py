"""CPU oracle for the packed multimodal DiT block (MiniMax-H3 shape).

TEST INFRASTRUCTURE ONLY.  This module is a plain, slow, fp64 numpy
restatement of what the hot path computes.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it.  It shares no code, tables or helpers with
the CUDA path under ``packed_multimodal_diffusion_b200/``, and the product
never imports it.

Sources, cited by page title and item:

* [mmh3]   "cortiq_engine/mmh3.rs" (docs.rs, cortiq-engine 0.5.72) -- the
           authority for layout, segment rows, the adaLN curve, the block,
           the stack and the output heads.
* [h3img]  "cortiq-engine 0.8.83 src/h3imagegen.rs" -- image-mode shapes.
* [siglip] "ffai-argus 0.7.0 src/siglip.rs" -- the SigLIP encoder layer.
* [enc]    "inferencelayer 0.2.1 src/encoder_cpu.rs" -- LayerNorm, rotary
           frequency formula, ragged attention.
* [zimage] "ollama x/imagegen/models/zimage/transformer.go" -- per-axis
           rotary frequency formula (corroboration only).

Every floating-point step runs in fp64 on inputs that the caller has already
rounded to the device storage type.  Library primitives used as steps:
``numpy.matmul`` / ``@`` (a dot product), ``numpy.exp``, ``numpy.sin``,
``numpy.cos``, ``numpy.tanh``.  There is no blocking, fusion or reordering
beyond what the definitions state.

Readings of points the pages leave open (numbered as in the design notes):

R1  adaLN output layout: the basis rows are [timestep slot][tag][chunk][H];
    slot s is evaluated at ts[s].
R2  Interpolation coordinates (i0, f) are computed in fp64.
R3  Rotary inverse frequencies are theta^(-i/k), theta = 10000, k = hd/8.
R6  Image mode: text [i,0,0], reference rows [text_len, h, w], target rows
    [text_len + 1, h, w]; every image row is tag VIDEO on the one clock.
R13 SigLIP LayerNorm eps = 1e-6 ("parity unpinned" for the eps value only).

Parity status: every function below is pinned by a ``-m "not gpu"`` test in
``tests/test_oracle_pins.py`` except the SigLIP LayerNorm eps value, which no
page prints (parity unpinned for that constant).
"""

from __future__ import annotations

import math

import numpy as np

# --------------------------------------------------------------------------
# constants  ([mmh3] module constants)
# --------------------------------------------------------------------------

#: Frames a video latent token spans, cycling with period 5 ([mmh3] constant
#: FRAME_PER_TOKEN), rescaled by 5/3 ([mmh3] FRAME_RESCALE).
FRAME_PER_TOKEN = (1.0, 4.0, 4.0, 4.0, 4.0)
FRAME_RESCALE = 5.0 / 3.0

#: Modality tags in adaLN row order ([mmh3] TAG_VIDEO / TAG_TEXT / TAG_AUDIO).
TAG_VIDEO, TAG_TEXT, TAG_AUDIO = 0, 1, 2
MODALITIES = 3
#: shift / scale / gate for attention, then for the MLP ([mmh3] EXPAND).
EXPAND = 6
#: Rows of the timestep-curve table ([mmh3] CURVE_GRID).
CURVE_GRID = 1025

#: Clocks: 0 = the video flow clock, 1 = the audio flow clock, 2 = the
#: visual condition clock (keyframe and reference-image rows), 3 = the audio
#: condition clock (reference audio rows).
CLOCK_VIDEO, CLOCK_AUDIO, CLOCK_COND, CLOCK_COND_AUDIO = 0, 1, 2, 3
#: Where condition rows sit on the schedule ([mmh3] VISUAL_COND_TIMESTEP,
#: AUDIO_COND_TIMESTEP; the model's cond_aug and cond_aug_audio).
VISUAL_COND_TIMESTEP = 0.999
AUDIO_COND_TIMESTEP = 1.0


# --------------------------------------------------------------------------
# flow-schedule remap  ([mmh3] "the flow-schedule remap")
# --------------------------------------------------------------------------

def time_shift_sigma(sigma: float, from_shift: float, to_shift: float) -> float:
    """sigma on the ``to_shift`` schedule at the same point of the shared
    base grid ([mmh3] ``time_shift_sigma``): first undo the ``from`` shift
    to get the base-grid value b, then apply the ``to`` shift."""
    b = sigma / (from_shift + sigma * (1.0 - from_shift))
    return to_shift * b / (1.0 + (to_shift - 1.0) * b)


def time_shift_slope(sigma: float, from_shift: float, to_shift: float) -> float:
    """d(sigma_to)/d(sigma_from) at the same base-grid point
    ([mmh3] ``time_shift_slope``)."""
    b = sigma / (from_shift + sigma * (1.0 - from_shift))
    return (to_shift * (1.0 + (from_shift - 1.0) * b) ** 2) / (
        from_shift * (1.0 + (to_shift - 1.0) * b) ** 2)


# --------------------------------------------------------------------------
# packed layout  ([mmh3] "the packed layout": Layout::build_full, t2va)
# --------------------------------------------------------------------------

def axis_from_sqrt_area(dim: int, patch: int, sqrt_area: float) -> list[float]:
    """Patch-centre coordinates along one spatial axis ([mmh3]
    ``axis_from_sqrt_area``): with ratio = dim / sqrt_area and n = dim/patch,
    entry i is (i * ratio / n + (1 - ratio) / 2) * 32."""
    ratio = dim / sqrt_area
    n = dim // patch
    return [(i * (ratio / n) + (1.0 - ratio) / 2.0) * 32.0 for i in range(n)]


def _audio_rows(cursor: float, t: int, w_low: float, w_high: float) -> list[tuple]:
    """Channel-major stereo audio rows ([mmh3] ``push_audio_grid``): channel 0
    then channel 1, each t frames long, h = 0, w pinned to the frame grid's
    low / high extreme."""
    rows = []
    for ch in range(2):
        w = w_low if ch == 0 else w_high
        for i in range(t):
            rows.append((cursor + i, 0.0, w))
    return rows


def layout_build_full(text_len: int, latent_t: int, lat_h: int, lat_w: int, audio_t: int,
                      frames=(), refs=(), text_tags=None) -> dict:
    """The packed layout ([mmh3] ``Layout::build_full``), step by step:

    * text rows (i, 0, 0); the segment table splits the prompt into runs of
      one modality tag (``text_tags``, default all TEXT), all on the video
      clock ([mmh3] ``forward``: text rows use t_v's index and their own tag);
    * the cursor starts at text_len; each reference, in order, advances it:
      ``("image", h, w)`` puts its own grid (``axis_from_sqrt_area`` of its
      own area) at the cursor, cursor + 1; ``("audio", t)`` puts t stereo
      frames at the cursor (w at the TARGET grid's extremes), cursor + t;
      ``("video", latent_t, h, w, audio_t)`` puts its soundtrack first (w at
      its own grid's extremes), then its frames with t stepping by
      5/3 * [1,4,4,4,4][k % 5], cursor + max(audio_t, summed spans);
    * keyframes ``(pixel_index, frame_count)`` on the target grid, not moving
      the cursor: the first frame at the cursor, the last one at cursor +
      spans - 5/3 (spans summed over the target's latent frames); any other
      frame is an error;
    * the target audio (stereo, target w extremes) and video from the cursor.

    Reference and keyframe rows are conditions ([mmh3] ``forward``):
    frames tag VIDEO on the visual condition clock, reference audio tag AUDIO
    on the audio condition clock.  Returns seq_len, frame_rows, segments
    (start, stop, tag, clock), kinds (the page's segment kind per segment)
    and pos [n, 3] float64."""
    area = math.sqrt(lat_h * lat_w)
    h_axis = axis_from_sqrt_area(lat_h, 2, area)
    w_axis = axis_from_sqrt_area(lat_w, 2, area)
    pos: list[tuple] = []
    segments, kinds = [], []

    def seg(start, tag, clock, kind):
        segments.append((start, len(pos), tag, clock))
        kinds.append(kind)

    tags = [TAG_TEXT] * text_len if text_tags is None else list(text_tags)
    run0 = 0
    for i in range(text_len):
        if i > 0 and tags[i] != tags[i - 1]:
            seg(run0, tags[i - 1], CLOCK_VIDEO, "Text")
            run0 = len(pos)
        pos.append((float(i), 0.0, 0.0))
    seg(run0, tags[-1], CLOCK_VIDEO, "Text")
    cursor = float(text_len)
    w_low_t, w_high_t = w_axis[0], w_axis[-1]
    for r in refs:
        if r[0] == "image":
            _, rh_, rw_ = r
            a = math.sqrt(rh_ * rw_)
            rh, rw = axis_from_sqrt_area(rh_, 2, a), axis_from_sqrt_area(rw_, 2, a)
            s0 = len(pos)
            pos += [(cursor, h, w) for h in rh for w in rw]
            seg(s0, TAG_VIDEO, CLOCK_COND, "RefImg")
            cursor += 1.0
        elif r[0] == "audio":
            t = r[1]
            if t > 0:
                s0 = len(pos)
                pos += _audio_rows(cursor, t, w_low_t, w_high_t)
                seg(s0, TAG_AUDIO, CLOCK_COND_AUDIO, "RefAudio")
            cursor += float(t)
        elif r[0] == "video":
            _, vt, rh_, rw_, rt = r
            a = math.sqrt(rh_ * rw_)
            rh, rw = axis_from_sqrt_area(rh_, 2, a), axis_from_sqrt_area(rw_, 2, a)
            if rt > 0:
                s0 = len(pos)
                pos += _audio_rows(cursor, rt, rw[0], rw[-1])
                seg(s0, TAG_AUDIO, CLOCK_COND_AUDIO, "RefAudio")
            s0 = len(pos)
            t_coord = cursor
            for k in range(vt):
                pos += [(t_coord, h, w) for h in rh for w in rw]
                t_coord += FRAME_RESCALE * FRAME_PER_TOKEN[k % 5]
            seg(s0, TAG_VIDEO, CLOCK_COND, "RefImg")
            spans = 0.0
            for k in range(vt):
                spans += FRAME_RESCALE * FRAME_PER_TOKEN[k % 5]
            cursor += max(float(rt), spans)
        else:
            raise ValueError(f"reference kind {r[0]!r}")
    spans = 0.0
    for k in range(latent_t):
        spans += FRAME_RESCALE * FRAME_PER_TOKEN[k % 5]
    for (pixel_index, frame_count) in frames:
        if pixel_index == 0:
            cond_t = cursor
        elif frame_count > 0 and pixel_index == frame_count - 1:
            cond_t = cursor + spans - FRAME_RESCALE
        else:
            raise ValueError("only the first and last frame can anchor a keyframe")
        s0 = len(pos)
        pos += [(cond_t, h, w) for h in h_axis for w in w_axis]
        seg(s0, TAG_VIDEO, CLOCK_COND, "Cond")
    a0 = len(pos)
    pos += _audio_rows(cursor, audio_t, w_low_t, w_high_t)
    seg(a0, TAG_AUDIO, CLOCK_AUDIO, "Audio")
    v0 = len(pos)
    t_coord = cursor
    for k in range(latent_t):
        pos += [(t_coord, h, w) for h in h_axis for w in w_axis]
        t_coord += FRAME_RESCALE * FRAME_PER_TOKEN[k % 5]
    seg(v0, TAG_VIDEO, CLOCK_VIDEO, "Video")
    return {
        "seq_len": len(pos),
        "frame_rows": len(h_axis) * len(w_axis),
        "segments": segments,
        "kinds": kinds,
        "pos": np.asarray(pos, dtype=np.float64).reshape(-1, 3),
    }


def layout_t2va(text_len: int, latent_t: int, lat_h: int, lat_w: int,
                audio_t: int) -> dict:
    """The text-to-video+audio layout ``[text | audio | video]``
    ([mmh3] ``Layout::t2va``: ``build_full`` with no keyframes or
    references).  Text uses the video clock, audio the audio clock, video the
    video clock."""
    return layout_build_full(text_len, latent_t, lat_h, lat_w, audio_t)


def layout_fl2va(text_len: int, latent_t: int, lat_h: int, lat_w: int, audio_t: int,
                 frames, text_tags=None) -> dict:
    """Keyframes between the text and the audio ([mmh3] ``Layout::fl2va``)."""
    return layout_build_full(text_len, latent_t, lat_h, lat_w, audio_t, frames=frames,
                             text_tags=text_tags)


def layout_ref2va(text_len: int, latent_t: int, lat_h: int, lat_w: int, audio_t: int,
                  refs, text_tags=None) -> dict:
    """References ahead of the target streams ([mmh3] ``Layout::ref2va``)."""
    return layout_build_full(text_len, latent_t, lat_h, lat_w, audio_t, refs=refs,
                             text_tags=text_tags)


def layout_image(text_len: int, ref_lat_h: int, ref_lat_w: int,
                 lat_h: int, lat_w: int) -> dict:
    """Image-mode layout ``[text | reference image | target image]``.

    Reading R6 (the pages call ``Layout::image`` but do not print it): the
    reference image follows the ``Ref::Image`` rule of [mmh3]
    ``build_full`` -- rows at the cursor's t with its own h/w grid, cursor
    advances by one -- and the target image takes the next t.  Every image
    row carries the VIDEO tag on the single (video) clock."""
    pos: list[tuple] = [(float(i), 0.0, 0.0) for i in range(text_len)]
    segments = [(0, text_len, TAG_TEXT, CLOCK_VIDEO)]
    cursor = float(text_len)
    for (lh, lw) in ((ref_lat_h, ref_lat_w), (lat_h, lat_w)):
        area = math.sqrt(lh * lw)
        hs = axis_from_sqrt_area(lh, 2, area)
        ws = axis_from_sqrt_area(lw, 2, area)
        s0 = len(pos)
        for h in hs:
            for w in ws:
                pos.append((cursor, h, w))
        segments.append((s0, len(pos), TAG_VIDEO, CLOCK_VIDEO))
        cursor += 1.0
    return {
        "seq_len": len(pos),
        "segments": segments,
        "pos": np.asarray(pos, dtype=np.float64).reshape(-1, 3),
    }


# --------------------------------------------------------------------------
# timesteps and per-token modulation rows  ([mmh3] ``forward``)
# --------------------------------------------------------------------------

def plan_timesteps(sigma_v: float, sigma_a: float, segments) -> tuple[list, dict]:
    """Distinct timesteps in ascending order and the slot of each clock.

    [mmh3] ``forward``: sigma_v is clamped to >= 1e-6, t_v = 1 - sigma_v,
    t_a = 1 - sigma_a; keyframe and reference-image rows sit at
    t_cond = max(t_v, VISUAL_COND_TIMESTEP), reference audio rows at
    t_cond_a = max(t_a, AUDIO_COND_TIMESTEP); the list of distinct timesteps
    is sorted and de-duplicated, and a row's adaLN slot is the position of
    its clock's timestep in that list.  Only clocks that some segment uses
    enter the list (image mode has one clock)."""
    sigma_v = max(sigma_v, 1e-6)
    t_v, t_a = 1.0 - sigma_v, 1.0 - sigma_a
    t_of_clock = {CLOCK_VIDEO: t_v, CLOCK_AUDIO: t_a,
                  CLOCK_COND: max(t_v, VISUAL_COND_TIMESTEP),
                  CLOCK_COND_AUDIO: max(t_a, AUDIO_COND_TIMESTEP)}
    used = sorted({seg[3] for seg in segments})
    ts = sorted({t_of_clock[c] for c in used})
    slot = {c: ts.index(t_of_clock[c]) for c in used}
    return ts, slot


def token_rows(segments, slot: dict, n: int) -> np.ndarray:
    """Per-token adaLN row = slot(clock) * MODALITIES + tag ([mmh3]
    ``forward``, "Per-token modulation row")."""
    rows = np.full(n, -1, dtype=np.int64)
    for (start, stop, tag, clock) in segments:
        rows[start:stop] = slot[clock] * MODALITIES + tag
    assert (rows >= 0).all(), "segments must cover every token"
    return rows


# --------------------------------------------------------------------------
# adaLN as a curve  ([mmh3] ``Adaln::eval``)
# --------------------------------------------------------------------------

def adaln_coords(table: np.ndarray, t: float) -> np.ndarray:
    """Rank-R curve coordinates at timestep t: p = clamp(t, 0, 1) * (G - 1),
    i0 = min(floor(p), G - 2), f = p - i0, and c the linear interpolation
    between table rows a = i0 and b = i0 + 1 at fraction f ([mmh3]
    ``Adaln::eval``).  Reading R2: fp64 throughout, and the interpolation is
    written (1 - f) a + f b so that it returns the node row exactly at both
    ends of an interval (t = 1 gives the last row, not a + (b - a))."""
    table = np.asarray(table, dtype=np.float64)
    g = table.shape[0]
    p = min(max(t, 0.0), 1.0) * (g - 1)
    i0 = min(int(math.floor(p)), g - 2)
    f = p - i0
    a, b = table[i0], table[i0 + 1]
    return (1.0 - f) * a + f * b


def adaln_eval(w: np.ndarray, b: np.ndarray, table: np.ndarray, ts,
               rows_per_slot: int) -> np.ndarray:
    """Modulation vectors for the distinct timesteps ``ts``.

    Reading R1: the basis ``w`` [slots * rows_per_slot, R] holds
    ``rows_per_slot`` = tags * chunks * H rows per timestep slot; slot s is
    ``w[s*rows_per_slot:(s+1)*rows_per_slot] @ c(ts[s]) + b[...]``.  The
    result is the concatenation over slots, i.e. a buffer of shape
    [len(ts) * tags, chunks * H] read at row ``slot * tags + tag``
    ([mmh3] ``Adaln::eval`` doc comment and ``modulate``)."""
    w = np.asarray(w, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    out = []
    for s, t in enumerate(ts):
        c = adaln_coords(table, t)
        lo, hi = s * rows_per_slot, (s + 1) * rows_per_slot
        out.append(w[lo:hi] @ c + b[lo:hi])
    return np.concatenate(out)


def block_mods(w, b, table, ts, hidden: int) -> np.ndarray:
    """A block's modulation buffer [len(ts) * 3, 6 * hidden]."""
    flat = adaln_eval(w, b, table, ts, MODALITIES * EXPAND * hidden)
    return flat.reshape(len(ts) * MODALITIES, EXPAND * hidden)


def final_mods(w, b, table, ts, hidden: int) -> np.ndarray:
    """The final layer's modulation buffer [len(ts), 2 * hidden]: one
    modality, chunks (shift, scale); the row is the timestep index
    ([mmh3] ``forward`` heads)."""
    flat = adaln_eval(w, b, table, ts, 2 * hidden)
    return flat.reshape(len(ts), 2 * hidden)


def chunk(mods_row: np.ndarray, e: int, hidden: int) -> np.ndarray:
    """Chunk e (0 shift_msa, 1 scale_msa, 2 gate_msa, 3 shift_mlp,
    4 scale_mlp, 5 gate_mlp) of a modulation row ([mmh3] ``modulate`` /
    ``residual``: chunk e starts at e * hidden)."""
    return mods_row[..., e * hidden:(e + 1) * hidden]


# --------------------------------------------------------------------------
# elementwise pieces  ([mmh3] rms_norm_into, silu, modulate, residual)
# --------------------------------------------------------------------------

def rms_norm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * g
    ([mmh3] ``rms_norm_into``)."""
    x = np.asarray(x, dtype=np.float64)
    inv = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return x * inv * np.asarray(g, dtype=np.float64)


def modulate(xn: np.ndarray, shift: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """x * (1 + scale) + shift ([mmh3] ``modulate``)."""
    return xn * (1.0 + scale) + shift


def silu(v: np.ndarray) -> np.ndarray:
    """v / (1 + exp(-v)) ([mmh3] ``silu``)."""
    return v / (1.0 + np.exp(-v))


# --------------------------------------------------------------------------
# qk-norm and 3-axis rotary embedding  ([mmh3] rope_angles, norm_rope_w)
# --------------------------------------------------------------------------

def rope_inv_freq(k: int, theta: float = 10000.0) -> np.ndarray:
    """Per-axis inverse frequencies theta^(-i/k), i < k (reading R3: the
    per-axis half-dimension formula of [enc] ``apply_rope`` and [zimage]
    ``prepareRoPE3D``; the checkpoint tensor itself is not printed)."""
    return theta ** (-np.arange(k, dtype=np.float64) / k)


def rope_angles(pos: np.ndarray, inv_freq: np.ndarray) -> np.ndarray:
    """[n, 3k] angles, axis-major: angle[axis * k + j] = pos[axis] *
    inv_freq[j] ([mmh3] ``rope_angles``).  As on that page, the frequencies
    are the model's f32 tensor (``dit.rope_inv_freq`` is read as f32), the
    product is taken in f64 from the f64 position, and each angle is stored
    as f32; the returned array holds those f32 values widened to f64."""
    pos = np.asarray(pos, dtype=np.float64)
    inv32 = np.asarray(inv_freq, dtype=np.float32).astype(np.float64)
    prod = pos[:, :, None] * inv32[None, None, :]
    return prod.astype(np.float32).astype(np.float64).reshape(pos.shape[0], -1)


def qk_norm_rope(v: np.ndarray, w: np.ndarray, angles: np.ndarray,
                 eps: float) -> np.ndarray:
    """Per-head RMSNorm (weight ``w`` [hd]) then the partial split-half
    rotation ([mmh3] ``norm_rope_w``): with P = angles.shape[1] pairs, head
    dims (j, j + P) turn by angle j for j < P; dims >= 2P are not rotated.

    ``v`` is [n, heads, hd]; ``angles`` is [n, P] (P = 0: no rotation)."""
    y = rms_norm(v, w, eps)
    npair = angles.shape[1]
    if npair == 0:
        return y
    c = np.cos(angles)[:, None, :]
    s = np.sin(angles)[:, None, :]
    lo = y[:, :, :npair].copy()
    hi = y[:, :, npair:2 * npair].copy()
    out = y.copy()
    out[:, :, :npair] = lo * c - hi * s
    out[:, :, npair:2 * npair] = lo * s + hi * c
    return out


# --------------------------------------------------------------------------
# attention  ([mmh3] ``attention`` host loop, ``softmax_inplace``)
# --------------------------------------------------------------------------

def softmax_rows(s: np.ndarray) -> np.ndarray:
    """Row softmax with the max subtracted and a den > 0 guard
    ([mmh3] ``softmax_inplace``)."""
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    den = np.sum(e, axis=-1, keepdims=True)
    return np.where(den > 0, e / np.where(den > 0, den, 1.0), e)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
              q_rows=None) -> np.ndarray:
    """Full bidirectional attention per head ([mmh3] ``attention``):
    S = (q * scale) k^T, P = softmax(S), O = P v.

    q, k, v are [n, heads, hd]; ``q_rows`` optionally selects which query
    rows to compute (all keys are always used).  Returns [len(q_rows), heads,
    hd]."""
    if q_rows is not None:
        q = q[q_rows]
    out = np.empty((q.shape[0], q.shape[1], v.shape[2]), dtype=np.float64)
    for h in range(q.shape[1]):
        s = (q[:, h, :] * scale) @ k[:, h, :].T
        out[:, h, :] = softmax_rows(s) @ v[:, h, :]
    return out


# --------------------------------------------------------------------------
# the block  ([mmh3] ``block_forward`` and ``ffn_tail``)
# --------------------------------------------------------------------------

def block_forward(p: dict, x: np.ndarray, mods, rows, pos, dims: dict,
                  sample_rows=None, keep: dict | None = None,
                  kv_cache: dict | None = None) -> np.ndarray:
    """One modulated DiT block ([mmh3] ``block_forward`` + ``ffn_tail``).

    ``p``: norm1, norm2 [H]; wqkv [3I, H] (rows [q | k | v], heads
    contiguous); wout [H, I]; q_norm, k_norm [hd]; wfc1 [2F, H] (rows
    [gate | up]); wfc2 [H, F].  No projection biases.
    ``mods`` [slots*3, 6H] or None (unmodulated, plain residual: the token
    refiner); ``rows`` [n] adaLN row per token; ``pos`` [n, 3] or None
    (unrotated).  ``dims``: hidden, heads, head_dim, ffn, eps, qk_eps,
    rope_k, rope_theta.

    ``sample_rows``: compute the output only for these token rows (k and v
    are still computed for every token, since attention reads all keys).
    ``keep``: if a dict, intermediates (xn1, q, k, v, attn, xmid, xn2, act)
    for the computed rows are stored in it.
    ``kv_cache``: if a dict, k (after qk-norm and rotation) and v of every
    token are stored in it by the first call and read back by later calls on
    the same x, so that a block can be computed in chunks of query rows with
    k and v computed once (the values are the same either way, up to the
    summation order the matrix product picks for a given row count).

    Returns x_out for the computed rows ([len(rows)] x H)."""
    H, nh, hd, F = dims["hidden"], dims["heads"], dims["head_dim"], dims["ffn"]
    eps, qk_eps = dims["eps"], dims["qk_eps"]
    I = nh * hd
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[0]
    sel = np.arange(n) if sample_rows is None else np.asarray(sample_rows)
    f64 = lambda a: np.asarray(a, dtype=np.float64)  # noqa: E731
    wqkv, wout, wfc1, wfc2 = f64(p["wqkv"]), f64(p["wout"]), f64(p["wfc1"]), f64(p["wfc2"])
    cached = kv_cache is not None and "k" in kv_cache
    # each token's modulation row [6H]: every token for k and v, or only the
    # computed rows when k and v come from the cache
    rows = np.asarray(rows)
    mr = None if mods is None else f64(mods)[rows[sel] if cached else rows]
    ms = None if mr is None else (mr if cached else mr[sel])

    # norm1 -> modulate(shift 0, scale 1)
    xr = x[sel] if cached else x
    xn1 = rms_norm(xr, p["norm1"], eps)
    if mr is not None:
        xn1 = modulate(xn1, chunk(mr, 0, H), chunk(mr, 1, H))
    xn1_sel = xn1 if cached else xn1[sel]
    if pos is None:
        ang_all = np.zeros((n, 0))
    else:
        ang_all = rope_angles(pos, rope_inv_freq(dims["rope_k"], dims["rope_theta"]))
    # qkv projection: q only where needed, k and v for every token
    q = (xn1_sel @ wqkv[:I].T).reshape(-1, nh, hd)
    q = qk_norm_rope(q, p["q_norm"], ang_all[sel], qk_eps)
    if cached:
        k, v = kv_cache["k"], kv_cache["v"]
    else:
        k = (xn1 @ wqkv[I:2 * I].T).reshape(n, nh, hd)
        v = (xn1 @ wqkv[2 * I:].T).reshape(n, nh, hd)
        k = qk_norm_rope(k, p["k_norm"], ang_all, qk_eps)
        if kv_cache is not None:
            kv_cache["k"], kv_cache["v"] = k, v
    o = attention(q, k, v, 1.0 / math.sqrt(hd)).reshape(-1, I)
    proj = o @ wout.T
    xs = x[sel]
    xmid = xs + (proj if ms is None else chunk(ms, 2, H) * proj)
    # ffn tail: norm2 -> modulate(3, 4) -> fc1 -> SwiGLU -> fc2 -> gate 5
    xn2 = rms_norm(xmid, p["norm2"], eps)
    if ms is not None:
        xn2 = modulate(xn2, chunk(ms, 3, H), chunk(ms, 4, H))
    gu = xn2 @ wfc1.T
    act = silu(gu[:, :F]) * gu[:, F:]
    down = act @ wfc2.T
    xout = xmid + (down if ms is None else chunk(ms, 5, H) * down)
    if keep is not None:
        keep.update(xn1=xn1_sel, q=q, k=k[sel], v=v[sel], attn=o, xmid=xmid,
                    xn2=xn2, act=act, rows=sel)
    return xout


def heads_forward(x_stream: np.ndarray, final_norm, fm_row, w, b,
                  eps: float) -> np.ndarray:
    """One output head ([mmh3] ``forward`` "heads"): RMSNorm(final_norm),
    then x * (1 + scale) + shift with the final adaLN row of the stream's
    timestep, then the linear map plus bias, then the sign flip (the model
    predicts toward the data)."""
    H = x_stream.shape[1]
    hn = rms_norm(x_stream, final_norm, eps)
    fm_row = np.asarray(fm_row, dtype=np.float64)
    hn = modulate(hn, fm_row[:H], fm_row[H:2 * H])
    y = hn @ np.asarray(w, dtype=np.float64).T + np.asarray(b, dtype=np.float64)
    return -y


# --------------------------------------------------------------------------
# SigLIP encoder layer  ([siglip] Layer::load / forward / finish_attention)
# --------------------------------------------------------------------------

def layer_norm(x: np.ndarray, g, b, eps: float) -> np.ndarray:
    """LayerNorm with a two-pass variance ([enc] ``layer_norm_rows``):
    (x - mean) / sqrt(var + eps) * g + b."""
    x = np.asarray(x, dtype=np.float64)
    mu = np.mean(x, axis=-1, keepdims=True)
    d = x - mu
    var = np.mean(d * d, axis=-1, keepdims=True)
    return d / np.sqrt(var + eps) * np.asarray(g, np.float64) + np.asarray(b, np.float64)


def gelu_tanh(x: np.ndarray) -> np.ndarray:
    """tanh-approximated GELU, 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))
    (Hendrycks & Gimpel; [siglip] ``gelu_one``, ``gelu_pytorch_tanh``)."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def vit_fold_scale(wq, bq, head_dim: int):
    """Fold the attention scale into the q projection ([siglip]
    ``Layer::load``): q * s = x (Wq s)^T + bq s with s = head_dim^-1/2."""
    s = head_dim ** -0.5
    return np.asarray(wq, np.float64) * s, np.asarray(bq, np.float64) * s


def vit_layer_forward(p: dict, x: np.ndarray, batch: int, seq: int, dims: dict,
                      images=None, keep: dict | None = None) -> np.ndarray:
    """One pre-norm SigLIP encoder layer over ``batch`` independent images
    of ``seq`` tokens ([siglip] ``Layer::forward`` / ``finish_attention``):

        y = x + (attn(LN1 x) Wo^T + bo)
        z = y + (gelu_tanh(LN2 y W1^T + b1) W2^T + b2)

    ``p["wqkv"]`` [3H, H] and ``p["bqkv"]`` [3H] already carry the attention
    scale in their q third (``vit_fold_scale``), so attention applies none.
    Attention runs within each image only.  ``images`` optionally restricts
    the computation to those image indices.  Returns [len(images)*seq, H]."""
    H, nh, hd, eps = dims["hidden"], dims["heads"], dims["head_dim"], dims["ln_eps"]
    f64 = lambda a: np.asarray(a, dtype=np.float64)  # noqa: E731
    x = f64(x).reshape(batch, seq, H)
    imgs = range(batch) if images is None else images
    outs = []
    for i in imgs:
        xi = x[i]
        hn = layer_norm(xi, p["ln1_g"], p["ln1_b"], eps)
        qkv = hn @ f64(p["wqkv"]).T + f64(p["bqkv"])
        q = qkv[:, :H].reshape(seq, nh, hd)
        k = qkv[:, H:2 * H].reshape(seq, nh, hd)
        v = qkv[:, 2 * H:].reshape(seq, nh, hd)
        o = attention(q, k, v, 1.0).reshape(seq, H)
        y = xi + (o @ f64(p["wo"]).T + f64(p["bo"]))
        h2 = layer_norm(y, p["ln2_g"], p["ln2_b"], eps)
        a = gelu_tanh(h2 @ f64(p["w1"]).T + f64(p["b1"]))
        z = y + (a @ f64(p["w2"]).T + f64(p["b2"]))
        if keep is not None:
            keep.setdefault("attn", []).append(o)
            keep.setdefault("y", []).append(y)
            keep.setdefault("act", []).append(a)
        outs.append(z)
    return np.concatenate(outs)


# --------------------------------------------------------------------------
# token refiner  ([mmh3] ``refine_text``)
# --------------------------------------------------------------------------

def refine_text(states: np.ndarray, cond_w, cond_b, blocks: list, refiner_norm,
                dims: dict, final_eps: float) -> np.ndarray:
    """Text states [n, text_dim] -> refined embeddings [n, H] ([mmh3]
    ``refine_text``): h = states cond_w^T + cond_b, then each refiner block
    unmodulated and unrotated (plain residuals), then RMSNorm with the
    refiner's final gain and eps."""
    h = np.asarray(states, np.float64) @ np.asarray(cond_w, np.float64).T + np.asarray(cond_b, np.float64)
    n = h.shape[0]
    for p in blocks:
        h = block_forward(p, h, None, np.zeros(n, dtype=np.int64), None, dims)
    return rms_norm(h, refiner_norm, final_eps)


# --------------------------------------------------------------------------
# stream (un)packing and the embed  ([mmh3] patchify_video, pack_audio, forward "embed")
# --------------------------------------------------------------------------

def patchify_video(x: np.ndarray) -> np.ndarray:
    """[C, T, H, W] -> [T*(H/2)*(W/2), 4C]: 2x2 spatial patches, each row
    ordered (channel, patch row p, patch column q) ([mmh3] ``patchify_video``,
    einsum nctrhpwq -> nthwcrpq)."""
    C, T, H, W = x.shape
    y = x.reshape(C, T, H // 2, 2, W // 2, 2)            # c t h p w q
    return y.transpose(1, 2, 4, 0, 3, 5).reshape(T * (H // 2) * (W // 2), 4 * C)


def unpatchify_video(rows: np.ndarray, C: int, T: int, H: int, W: int) -> np.ndarray:
    """The inverse of ``patchify_video`` ([mmh3] ``unpatchify_video``)."""
    y = np.asarray(rows).reshape(T, H // 2, W // 2, C, 2, 2)   # t h w c p q
    return y.transpose(3, 0, 1, 4, 2, 5).reshape(C, T, H, W)


def pack_audio(x: np.ndarray) -> np.ndarray:
    """[C, 2, T] -> [2T, C], channel-major: stereo channel 0's frames then
    channel 1's ([mmh3] ``pack_audio``)."""
    C, two, T = x.shape
    return np.asarray(x).transpose(1, 2, 0).reshape(2 * T, C)


def unpack_audio(rows: np.ndarray, C: int, T: int) -> np.ndarray:
    """The inverse of ``pack_audio`` ([mmh3] ``unpack_audio``)."""
    return np.asarray(rows).reshape(2, T, C).transpose(2, 0, 1)


def embed(layout: dict, text: np.ndarray, video: np.ndarray, audio: np.ndarray,
          w_video, b_video, w_audio, b_audio, cond: list = ()) -> np.ndarray:
    """The packed hidden states of one denoise evaluation ([mmh3] ``forward``
    "embed").  The first text-tag segment takes the refined text rows; the
    LAST video-tag segment (the target) takes the video latents, patchified
    and projected (+ bias); the last audio-tag segment takes the audio
    latents, packed and projected (+ bias).  Every other video-tag segment is
    a condition frame: ``cond[i]`` ([C, 1, h, w], noise blend already applied
    by the caller) goes through the same patch projection, in segment order.
    Rows of no segment stay zero."""
    n = layout["seq_len"]
    Hd = np.asarray(w_video).shape[0]
    h = np.zeros((n, Hd))
    segs = layout["segments"]
    t_idx = [k for k, s in enumerate(segs) if s[2] == TAG_TEXT]
    v_idx = [k for k, s in enumerate(segs) if s[2] == TAG_VIDEO]
    a_idx = [k for k, s in enumerate(segs) if s[2] == TAG_AUDIO]
    wv, bv = np.asarray(w_video, np.float64), np.asarray(b_video, np.float64)
    if t_idx:
        a, b = segs[t_idx[0]][:2]
        h[a:b] = np.asarray(text, np.float64)[: b - a]
    if v_idx:
        a, b = segs[v_idx[-1]][:2]
        h[a:b] = patchify_video(np.asarray(video, np.float64)) @ wv.T + bv
        for i, k in enumerate(v_idx[:-1]):
            a, b = segs[k][:2]
            h[a:b] = patchify_video(np.asarray(cond[i], np.float64)) @ wv.T + bv
    if a_idx:
        a, b = segs[a_idx[-1]][:2]
        h[a:b] = pack_audio(np.asarray(audio, np.float64)) @ np.asarray(w_audio, np.float64).T \
            + np.asarray(b_audio, np.float64)
    return h


def denoise_forward(layout: dict, text, video, audio, embed_w: tuple, blocks: list, heads: dict,
                    sigma_v: float, sigma_a: float, dims: dict, cond: list = ()):
    """One denoise evaluation ([mmh3] ``forward``): the embed, every block
    (modulated, rotated by the layout's positions), the output heads on the
    target video and audio segments, then the head rows unpatchified /
    unpacked.  ``embed_w`` = (w_video, b_video, w_audio, b_audio).  Returns
    (video velocity [C, T, h, w], audio velocity [C, 2, T]), each on its own
    clock and negated by the heads."""
    segs, n = layout["segments"], layout["seq_len"]
    H = dims["hidden"]
    h = embed(layout, text, video, audio, *embed_w, cond=cond)
    ts, slot = plan_timesteps(sigma_v, sigma_a, segs)
    rows = token_rows(segs, slot, n)
    for p in blocks:
        mods = block_mods(p["adaln_w"], p["adaln_b"], p["adaln_table"], ts, H)
        h = block_forward(p, h, mods, rows, layout["pos"], dims)
    fm = final_mods(heads["adaln_w"], heads["adaln_b"], heads["adaln_table"], ts, H)
    v_seg = [s for s in segs if s[2] == TAG_VIDEO][-1]
    a_seg = [s for s in segs if s[2] == TAG_AUDIO][-1]
    out = []
    for (a, b, _tag, clock), key in ((v_seg, "video"), (a_seg, "audio")):
        out.append(heads_forward(h[a:b], heads["final_norm"], fm[slot[clock]],
                                 heads[f"w_{key}"], heads[f"b_{key}"], dims["eps"]))
    C, T, lh, lw = np.asarray(video).shape
    Ca, _, Ta = np.asarray(audio).shape
    return unpatchify_video(out[0], C, T, lh, lw), unpack_audio(out[1], Ca, Ta)
