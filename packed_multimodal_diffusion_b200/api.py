"""Python binding of the C ABI for torch tensors (marshalling only: every step
of the path runs in libmmh3.so's kernels on the caller's current CUDA
stream).  Device tensors must be contiguous CUDA tensors; PyTorch provides
device memory and streams, nothing else."""

from __future__ import annotations

import ctypes as C
from dataclasses import dataclass

import numpy as np
import torch

from . import _lib
from ._lib import (MMH3_BF16, MMH3_F32, MMH3_REF_AUDIO, MMH3_REF_IMAGE, MMH3_REF_VIDEO, MMH3_STREAM_AUDIO,
                   MMH3_STREAM_VIDEO, BlockWeights, Dims, EmbedInputs, EmbedWeights, HeadWeights, Keyframe, Ref,
                   Segment, VitDims, VitWeights, check, load)

__all__ = ["Dims", "Segment", "make_dims", "segments", "layout_t2va", "layout_image",
           "plan_timesteps", "time_shift_sigma", "resolve_rows", "adaln_modulation",
           "prepare_block_weights", "prepare_fc1", "workspace_size", "attention", "attention_ws", "BlockParams", "HeadParams",
           "block_forward", "stack_forward", "block_forward_host", "block_cp_begin", "block_cp_end", "refine_workspace_size", "refine_text",
           "patch_embed_workspace_size", "patch_embed", "embed_workspace_size", "embed",
           "unpatchify_video", "unpack_audio", "forward_workspace_size", "forward", "VitParams", "vit_fold_qkv", "vit_workspace_size",
           "vit_layer_forward", "vit_dims", "layout_fl2va", "layout_ref2va", "block_forward_noalloc",
           "workspace_regions", "device_status", "status_sync", "set_check", "selftest_wait_timeout",
           "set_wait_limit_ns", "launch_count", "prof_enable", "prof_reset", "prof_collect",
           "prof_collect_kernels", "MMH3_BF16", "MMH3_F32"]


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("expected a contiguous CUDA tensor")
    return t.data_ptr()


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return MMH3_BF16
    if dt == torch.float32:
        return MMH3_F32
    raise ValueError(f"unsupported activation dtype {dt}")


def make_dims(hidden, heads, head_dim, ffn, act_dtype=torch.bfloat16, rank=24, grid=1025,
              eps=1e-5, qk_eps=1e-5, rope_theta=10000.0) -> Dims:
    return Dims(hidden, heads, head_dim, ffn, rank, grid, head_dim // 8, eps, qk_eps, rope_theta,
                _dtype_code(act_dtype))


def segments(segs) -> C.Array:
    """(start, stop, tag, clock) tuples -> a ctypes array of mmh3_segment."""
    arr = (Segment * len(segs))()
    for i, (a, b, tag, clock) in enumerate(segs):
        arr[i].start, arr[i].stop, arr[i].tag, arr[i].clock = a, b, tag, clock
    return arr


def _seg_tuples(arr, n) -> list[tuple]:
    return [(arr[i].start, arr[i].stop, arr[i].tag, arr[i].clock) for i in range(n)]


def time_shift_sigma(sigma: float, from_shift: float, to_shift: float) -> float:
    return load().mmh3_time_shift_sigma(sigma, from_shift, to_shift)


def _layout(fn, *args):
    segs = (Segment * 16)()
    nseg, n = C.c_int(), C.c_int()
    check(fn(*args, segs, C.byref(nseg), None, 0, C.byref(n)))
    pos = np.zeros((n.value, 3), dtype=np.float32)
    check(fn(*args, segs, C.byref(nseg), pos.ctypes.data_as(C.POINTER(C.c_float)), n.value,
             C.byref(n)))
    return _seg_tuples(segs, nseg.value), pos


def layout_t2va(text_len, latent_t, lat_h, lat_w, audio_t):
    """-> (segments [(start, stop, tag, clock)], pos float32 [n, 3])."""
    return _layout(load().mmh3_layout_t2va, text_len, latent_t, lat_h, lat_w, audio_t)


def layout_image(text_len, ref_lat_h, ref_lat_w, lat_h, lat_w):
    return _layout(load().mmh3_layout_image, text_len, ref_lat_h, ref_lat_w, lat_h, lat_w)


def _layout_cap(fn, *args):
    """Layouts whose segment count varies (keyframes, references): segment
    capacity 16, positions queried first."""
    segs = (Segment * 16)()
    nseg, n = C.c_int(), C.c_int()
    check(fn(*args, segs, 16, C.byref(nseg), None, 0, C.byref(n)))
    pos = np.zeros((n.value, 3), dtype=np.float32)
    check(fn(*args, segs, 16, C.byref(nseg), pos.ctypes.data_as(C.POINTER(C.c_float)), n.value, C.byref(n)))
    return _seg_tuples(segs, nseg.value), pos


def _tags(text_tags):
    if text_tags is None:
        return None
    return (C.c_uint8 * len(text_tags))(*text_tags)


def layout_fl2va(text_len, latent_t, lat_h, lat_w, audio_t, frames, text_tags=None):
    """frames: [(pixel_index, frame_count)]; text_tags: per-token modality
    tags of the prompt (None: all text)."""
    kf = (Keyframe * max(1, len(frames)))(*[Keyframe(a, b) for a, b in frames])
    return _layout_cap(load().mmh3_layout_fl2va, text_len, latent_t, lat_h, lat_w, audio_t, kf, len(frames),
                       _tags(text_tags))


def layout_ref2va(text_len, latent_t, lat_h, lat_w, audio_t, refs, text_tags=None):
    """refs: [("image", lat_h, lat_w) | ("audio", t) | ("video", latent_t, lat_h, lat_w, audio_t)]."""
    arr = (Ref * max(1, len(refs)))()
    for i, r in enumerate(refs):
        if r[0] == "image":
            arr[i] = Ref(MMH3_REF_IMAGE, r[1], r[2], 0, 0)
        elif r[0] == "audio":
            arr[i] = Ref(MMH3_REF_AUDIO, 0, 0, 0, r[1])
        else:
            arr[i] = Ref(MMH3_REF_VIDEO, r[2], r[3], r[1], r[4])
    return _layout_cap(load().mmh3_layout_ref2va, text_len, latent_t, lat_h, lat_w, audio_t, arr, len(refs),
                       _tags(text_tags))


def plan_timesteps(segs, n, sigma_v, sigma_a):
    arr = segments(segs)
    ts = (C.c_double * 4)()
    nts = C.c_int()
    rows = (C.c_int * len(segs))()
    check(load().mmh3_plan_timesteps(arr, len(segs), n, sigma_v, sigma_a, ts, C.byref(nts), rows))
    return list(ts)[: nts.value], list(rows)


def resolve_rows(segs, n, sigma_v, sigma_a, rows_out: torch.Tensor) -> None:
    check(load().mmh3_resolve_rows(segments(segs), len(segs), n, sigma_v, sigma_a,
                                   _ptr(rows_out), _stream()))


def adaln_modulation(dims: Dims, w, b, table, rows_per_slot, segs, n, sigma_v, sigma_a,
                     out: torch.Tensor) -> int:
    nts = C.c_int()
    check(load().mmh3_adaln_modulation(C.byref(dims), _ptr(w), _ptr(b), _ptr(table), rows_per_slot,
                                       segments(segs), len(segs), n, sigma_v, sigma_a, _ptr(out),
                                       C.byref(nts), _stream()))
    return nts.value


def prepare_block_weights(dims: Dims, fc1_gate_up: torch.Tensor, out: torch.Tensor) -> None:
    """fc1 [gate | up] -> the fused fc1+SwiGLU kernel's tile order."""
    check(load().mmh3_prepare_block_weights(C.byref(dims), _ptr(fc1_gate_up), _ptr(out), _stream()))


def prepare_fc1(dims: Dims, fc1_gate_up: torch.Tensor, out: torch.Tensor) -> None:
    check(load().mmh3_prepare_fc1(C.byref(dims), _ptr(fc1_gate_up), _ptr(out), _stream()))


def workspace_size(dims: Dims, n: int) -> int:
    v = C.c_size_t()
    check(load().mmh3_workspace_size(C.byref(dims), n, C.byref(v)))
    return v.value


def attention(qkv: torch.Tensor, n_seq: int, seq: int, heads: int, head_dim: int, scale: float,
              out: torch.Tensor) -> None:
    check(load().mmh3_attention(_ptr(qkv), n_seq, seq, heads, head_dim, _dtype_code(qkv.dtype),
                                scale, _ptr(out), _stream()))


def attention_ws(qkv: torch.Tensor, n_seq: int, seq: int, heads: int, head_dim: int, scale: float,
                 out: torch.Tensor, scratch: torch.Tensor | None) -> None:
    """attention with a scratch region that lets the last wave be split."""
    nbytes = 0 if scratch is None else scratch.numel() * scratch.element_size()
    check(load().mmh3_attention_ws(_ptr(qkv), n_seq, seq, heads, head_dim, _dtype_code(qkv.dtype), scale,
                                   _ptr(out), _ptr(scratch), nbytes, _stream()))


@dataclass
class BlockParams:
    """Device tensors of one block (fc1 already in the fused kernel's tile
    order, see prepare_fc1) and the matching C struct."""
    tensors: dict

    def struct(self) -> BlockWeights:
        t = self.tensors
        return BlockWeights(*[_ptr(t.get(k)) for k in ("norm1", "norm2", "wqkv", "wout", "q_norm",
                                                        "k_norm", "wfc1_tiled", "wfc2", "adaln_w",
                                                        "adaln_b", "adaln_table")])

    @staticmethod
    def from_host(dims: Dims, w: dict, device="cuda") -> "BlockParams":
        """Copy a host weight dict (natural layouts) to the device and tile
        fc1 for the fused SwiGLU kernel."""
        t = {k: v.to(device).contiguous() for k, v in w.items() if k != "wfc1"}
        fc1 = w["wfc1"].to(device).contiguous()
        t["wfc1_tiled"] = torch.empty_like(fc1)
        prepare_block_weights(dims, fc1, t["wfc1_tiled"])
        return BlockParams(t)


@dataclass
class HeadParams:
    tensors: dict

    def struct(self) -> HeadWeights:
        t = self.tensors
        return HeadWeights(*[_ptr(t.get(k)) for k in ("final_norm", "adaln_w", "adaln_b",
                                                       "adaln_table", "w_video", "b_video",
                                                       "w_audio", "b_audio")],
                           t["w_video"].shape[0], t["w_audio"].shape[0])

    @staticmethod
    def from_host(w: dict, device="cuda") -> "HeadParams":
        return HeadParams({k: v.to(device).contiguous() for k, v in w.items()})


def block_forward(dims: Dims, params: BlockParams, x: torch.Tensor, segs, pos: torch.Tensor | None,
                  sigma_v: float, sigma_a: float, workspace: torch.Tensor,
                  modulated: bool = True, mods: torch.Tensor | None = None) -> None:
    """In place on x [n, H] fp32.  ``mods``: an optional [T_s*3, 6H] fp32
    device modulation used instead of the block's adaLN curve."""
    st = params.struct()
    check(load().mmh3_block_forward(C.byref(dims), C.byref(st), _ptr(x), x.shape[0],
                                    segments(segs), len(segs), _ptr(pos), sigma_v, sigma_a,
                                    1 if modulated else 0, _ptr(mods), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream()))


def block_forward_noalloc(dims: Dims, params: BlockParams, x: torch.Tensor, segs,
                          pos: torch.Tensor | None, sigma_v: float, sigma_a: float,
                          modulated: bool = True) -> None:
    """mmh3_block_forward on the library's fixed device scratch (no
    workspace argument, nothing allocated by the call); in place on x."""
    st = params.struct()
    check(load().mmh3_block_forward_noalloc(C.byref(dims), C.byref(st), _ptr(x), x.shape[0],
                                            segments(segs), len(segs), _ptr(pos), sigma_v, sigma_a,
                                            1 if modulated else 0, _stream()))


def stack_forward(dims: Dims, blocks: list, heads: HeadParams | None, x: torch.Tensor, segs,
                  pos, sigma_v, sigma_a, out_video, out_audio, workspace) -> None:
    arr = (BlockWeights * max(1, len(blocks)))(*[b.struct() for b in blocks])
    hs = heads.struct() if heads is not None else None
    check(load().mmh3_stack_forward(C.byref(dims), arr, len(blocks),
                                    C.byref(hs) if hs is not None else None, _ptr(x), x.shape[0],
                                    segments(segs), len(segs), _ptr(pos), sigma_v, sigma_a,
                                    _ptr(out_video), _ptr(out_audio), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream()))


# ---------------------------------------------------- block on host buffers
def _host_ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if t.is_cuda or not t.is_contiguous() or not t.is_pinned():
        raise ValueError("expected a contiguous pinned host tensor")
    return t.data_ptr()


# Device slots of the host-buffer block (MMH3_HOST_SLOTS in mmh3.h).
HOST_SLOTS = 3


def block_forward_host(dims: Dims, params: BlockParams, x_in: torch.Tensor, x_out: torch.Tensor,
                       segs, pos: torch.Tensor | None, sigma_v: float, sigma_a: float, slot: int,
                       x_dev: torch.Tensor, pos_dev: torch.Tensor | None, workspace: torch.Tensor,
                       copy_in: torch.cuda.Stream, copy_out: torch.cuda.Stream) -> None:
    """One block from pinned host x_in (and pos) to pinned host x_out,
    through device slot `slot` (0 .. HOST_SLOTS - 1, one x_dev / pos_dev per
    slot; rotate them); copies on copy_in / copy_out, the block on the
    current stream.  Returns without waiting."""
    st = params.struct()
    check(load().mmh3_block_forward_host(C.byref(dims), C.byref(st), _host_ptr(x_in), _host_ptr(x_out),
                                         x_in.shape[0], segments(segs), len(segs), _host_ptr(pos),
                                         sigma_v, sigma_a, slot, _ptr(x_dev), _ptr(pos_dev),
                                         _ptr(workspace), workspace.numel() * workspace.element_size(),
                                         _stream(), copy_in.cuda_stream, copy_out.cuda_stream))


# ------------------------------------------------ block over a sequence shard
def block_cp_begin(dims: Dims, params: BlockParams, x: torch.Tensor, segs, pos, sigma_v: float,
                   sigma_a: float, kv_out: torch.Tensor, workspace: torch.Tensor,
                   modulated: bool = True) -> None:
    """The shard's block up to the qkv GEMM; its K|V rows go to kv_out
    [n, 2*inner] bf16.  segs are the shard's (rows from its first row)."""
    st = params.struct()
    check(load().mmh3_block_cp_begin(C.byref(dims), C.byref(st), _ptr(x), x.shape[0], segments(segs),
                                     len(segs), _ptr(pos), sigma_v, sigma_a, 1 if modulated else 0,
                                     _ptr(kv_out), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream()))


def block_cp_end(dims: Dims, params: BlockParams, x: torch.Tensor, segs, sigma_v: float,
                 sigma_a: float, kv_all: torch.Tensor, n_kv: int, workspace: torch.Tensor,
                 modulated: bool = True) -> None:
    """The rest of the shard's block against the gathered K|V rows (the first
    n_kv rows of kv_all); in place on x.  Same workspace as begin."""
    st = params.struct()
    check(load().mmh3_block_cp_end(C.byref(dims), C.byref(st), _ptr(x), x.shape[0], segments(segs),
                                   len(segs), sigma_v, sigma_a, 1 if modulated else 0, _ptr(kv_all),
                                   n_kv, _ptr(workspace), workspace.numel() * workspace.element_size(),
                                   _stream()))


# ------------------------------------------------ token refiner, embed, unpack
def refine_workspace_size(dims: Dims, n: int) -> int:
    b = C.c_size_t(0)
    check(load().mmh3_refine_workspace_size(C.byref(dims), n, C.byref(b)))
    return b.value


def refine_text(dims: Dims, states: torch.Tensor, cond_w: torch.Tensor, cond_b: torch.Tensor,
                blocks: list, refiner_norm: torch.Tensor, final_eps: float, out: torch.Tensor,
                workspace: torch.Tensor) -> None:
    """states [n, text_dim] act dtype -> out [n, H] fp32 (the token refiner)."""
    arr = (BlockWeights * max(1, len(blocks)))(*[b.struct() for b in blocks])
    check(load().mmh3_refine_text(C.byref(dims), _ptr(states), states.shape[0], states.shape[1],
                                  _ptr(cond_w), _ptr(cond_b), arr, len(blocks), _ptr(refiner_norm),
                                  final_eps, _ptr(out), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream()))


def _stream_args(kind: int, latents: torch.Tensor):
    if kind == MMH3_STREAM_VIDEO:
        c, t, h, w = latents.shape
        return c, t, h, w
    c, two, t = latents.shape
    if two != 2:
        raise ValueError("audio latents must be [C, 2, T]")
    return c, t, 0, 0


def patch_embed_workspace_size(dims: Dims, kind: int, latents_shape) -> int:
    b = C.c_size_t(0)
    if kind == MMH3_STREAM_VIDEO:
        c, t, h, w = latents_shape
    else:
        c, _, t = latents_shape
        h = w = 0
    check(load().mmh3_patch_embed_workspace_size(C.byref(dims), kind, c, t, h, w, C.byref(b)))
    return b.value


def patch_embed(dims: Dims, kind: int, latents: torch.Tensor, w: torch.Tensor, b: torch.Tensor,
                x_rows: torch.Tensor, workspace: torch.Tensor) -> None:
    """One stream's latents -> x_rows [rows, H] fp32 (patchify or pack, then
    the projection with bias)."""
    c, t, h, wd = _stream_args(kind, latents)
    check(load().mmh3_patch_embed(C.byref(dims), kind, _ptr(latents), c, t, h, wd, _ptr(w), _ptr(b),
                                  _ptr(x_rows), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream()))


def _embed_inputs(text, video, audio, cond):
    cond = list(cond or [])
    arr = (C.c_void_p * max(1, len(cond)))(*[_ptr(z) for z in cond])
    cv, tv, lh, lw = video.shape if video is not None else (1, 0, 2, 2)
    ca, _, ta = audio.shape if audio is not None else (1, 2, 0)
    ins = EmbedInputs(_ptr(text), _ptr(video), cv, tv, lh, lw, _ptr(audio), ca, ta,
                      C.cast(arr, C.POINTER(C.c_void_p)), len(cond))
    return ins, arr


def embed_workspace_size(dims: Dims, text, video, audio, cond=()) -> int:
    ins, _keep = _embed_inputs(text, video, audio, cond)
    b = C.c_size_t(0)
    check(load().mmh3_embed_workspace_size(C.byref(dims), C.byref(ins), C.byref(b)))
    return b.value


def embed(dims: Dims, segs, n: int, text, video, audio, w_video, b_video, w_audio, b_audio,
          x: torch.Tensor, workspace: torch.Tensor, cond=()) -> None:
    """The packed hidden states x [n, H] fp32 of one denoise evaluation."""
    ins, _keep = _embed_inputs(text, video, audio, cond)
    ew = EmbedWeights(_ptr(w_video), _ptr(b_video), _ptr(w_audio), _ptr(b_audio))
    check(load().mmh3_embed(C.byref(dims), segments(segs), len(segs), n, C.byref(ins), C.byref(ew),
                            _ptr(x), _ptr(workspace), workspace.numel() * workspace.element_size(),
                            _stream()))


def forward_workspace_size(dims: Dims, n: int, text, video, audio, cond=()) -> int:
    ins, _keep = _embed_inputs(text, video, audio, cond)
    b = C.c_size_t(0)
    check(load().mmh3_forward_workspace_size(C.byref(dims), n, C.byref(ins), C.byref(b)))
    return b.value


def forward(dims: Dims, segs, n: int, pos, sigma_v: float, sigma_a: float, text, video, audio,
            embed_w: tuple, blocks: list, heads: "HeadParams", x: torch.Tensor,
            video_out: torch.Tensor | None, audio_out: torch.Tensor | None,
            workspace: torch.Tensor, cond=()) -> None:
    """One denoise evaluation: embed -> blocks -> heads -> unpatchify /
    unpack.  embed_w = (w_video, b_video, w_audio, b_audio)."""
    ins, _keep = _embed_inputs(text, video, audio, cond)
    ew = EmbedWeights(*[_ptr(t) for t in embed_w])
    arr = (BlockWeights * max(1, len(blocks)))(*[b.struct() for b in blocks])
    hs = heads.struct()
    check(load().mmh3_forward(C.byref(dims), segments(segs), len(segs), n, _ptr(pos), sigma_v,
                              sigma_a, C.byref(ins), C.byref(ew), arr, len(blocks), C.byref(hs),
                              _ptr(x), _ptr(video_out), _ptr(audio_out), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _stream()))


def unpatchify_video(rows: torch.Tensor, channels: int, frames: int, lat_h: int, lat_w: int,
                     out: torch.Tensor) -> None:
    check(load().mmh3_unpatchify_video(_ptr(rows), channels, frames, lat_h, lat_w, _ptr(out),
                                       _stream()))


def unpack_audio(rows: torch.Tensor, channels: int, frames: int, out: torch.Tensor) -> None:
    check(load().mmh3_unpack_audio(_ptr(rows), channels, frames, _ptr(out), _stream()))


# -------------------------------------------------------------- encoder layer
def vit_dims(hidden, heads, head_dim, mlp, ln_eps=1e-6) -> VitDims:
    return VitDims(hidden, heads, head_dim, mlp, ln_eps)


@dataclass
class VitParams:
    tensors: dict

    def struct(self) -> VitWeights:
        t = self.tensors
        return VitWeights(*[_ptr(t[k]) for k in ("ln1_g", "ln1_b", "wqkv", "bqkv", "wo", "bo",
                                                  "ln2_g", "ln2_b", "w1", "b1", "w2", "b2")])

    @staticmethod
    def from_host(dims: VitDims, w: dict, device="cuda") -> "VitParams":
        t = {k: v.to(device).contiguous() for k, v in w.items()}
        H = dims.hidden
        t["wqkv"] = torch.empty((3 * H, H), dtype=torch.bfloat16, device=device)
        t["bqkv"] = torch.empty((3 * H,), dtype=torch.float32, device=device)
        vit_fold_qkv(dims, t["wq"], t["wk"], t["wv"], t["bq"], t["bk"], t["bv"], t["wqkv"],
                     t["bqkv"])
        return VitParams(t)


def vit_fold_qkv(dims: VitDims, wq, wk, wv, bq, bk, bv, wqkv, bqkv) -> None:
    check(load().mmh3_vit_fold_qkv(C.byref(dims), _ptr(wq), _ptr(wk), _ptr(wv), _ptr(bq), _ptr(bk),
                                   _ptr(bv), _ptr(wqkv), _ptr(bqkv), _stream()))


def vit_workspace_size(dims: VitDims, batch: int, seq: int) -> int:
    v = C.c_size_t()
    check(load().mmh3_vit_workspace_size(C.byref(dims), batch, seq, C.byref(v)))
    return v.value


def vit_layer_forward(dims: VitDims, params: VitParams, x: torch.Tensor, batch: int, seq: int,
                      workspace: torch.Tensor) -> None:
    st = params.struct()
    check(load().mmh3_vit_layer_forward(C.byref(dims), C.byref(st), _ptr(x), batch, seq,
                                        _ptr(workspace),
                                        workspace.numel() * workspace.element_size(), _stream()))


# ---------------------------------------------------------------- diagnostics
def device_status() -> tuple[int, int]:
    """Synchronise the current stream; return (code, site) of a recorded
    bounded-wait timeout, raising Mmh3Error(MMH3_ERR_TIMEOUT) if one was."""
    code, site = C.c_int(), C.c_int()
    check(load().mmh3_device_status(_stream(), C.byref(code), C.byref(site)))
    return code.value, site.value


def status_sync() -> int:
    """Synchronise the current stream and return the device status code
    (0 = none), raising Mmh3Error(MMH3_ERR_TIMEOUT) if a kernel gave up."""
    code = C.c_int()
    check(load().mmh3_status_sync(_stream(), C.byref(code)))
    return code.value


def selftest_wait_timeout(limit_ns: int) -> int:
    """Run the bounded-wait self test; returns the status code (7 expected)."""
    return load().mmh3_selftest_wait_timeout(limit_ns, _stream())


PROF_SLOTS = ("norm+mod", "qkv gemm", "qknorm+rope", "attention", "out gemm", "fc1 gemm",
              "swiglu", "fc2 gemm", "residual")


def prof_enable(on: bool = True) -> None:
    load().mmh3_prof_enable(1 if on else 0)


def prof_reset() -> None:
    load().mmh3_prof_reset()


def prof_collect() -> tuple[dict, int]:
    """Cumulative per-phase device milliseconds and the number of blocks."""
    ms = (C.c_double * 9)()
    nb = C.c_long()
    check(load().mmh3_prof_collect(ms, 9, C.byref(nb)))
    return dict(zip(PROF_SLOTS, list(ms))), nb.value


PROF_KERNELS = ("prologue", "norm1", "qkv gemm", "attention", "out gemm", "norm2", "fc1 gemm",
                "fc2 gemm")


def prof_collect_kernels() -> dict:
    """Cumulative device milliseconds and launch counts per kernel id
    (MMH3_PROF_K_*): {name: (ms, calls)}."""
    n = len(PROF_KERNELS)
    ms = (C.c_double * n)()
    calls = (C.c_long * n)()
    check(load().mmh3_prof_collect_kernels(ms, calls, n))
    return {k: (ms[i], calls[i]) for i, k in enumerate(PROF_KERNELS)}


def launch_count() -> int:
    """Kernels launched by the library in this process so far."""
    return int(load().mmh3_launch_count())


def set_check(on: int) -> None:
    """The check mode: 1 on, 0 off, -1 the environment's MMH3_CHECK."""
    load().mmh3_set_check(on)


def set_wait_limit_ns(ns: int) -> None:
    load().mmh3_set_wait_limit_ns(ns)


def workspace_regions(dims: Dims, n: int, ws: torch.Tensor) -> dict:
    """Views of the workspace regions (layout of mmh3_workspace_size) for
    inspecting a block's intermediates."""
    H, I, F = dims.hidden, dims.heads * dims.head_dim, dims.ffn
    act = torch.bfloat16 if dims.act_dtype == MMH3_BF16 else torch.float32
    es = 2 if dims.act_dtype == MMH3_BF16 else 4
    a256 = lambda v: (v + 255) // 256 * 256  # noqa: E731
    sizes = [("mods", 2 * 3 * 6 * H * 4, torch.float32, (6, 6 * H)),
             ("cs", n * 3 * dims.rope_k * 8, torch.float32, (3 * dims.rope_k, n, 2)),
             ("xn1", n * H * es, act, (n, H)), ("qkv", n * 3 * I * es, act, (n, 3 * I)),
             ("attn", n * I * es, act, (n, I)), ("xn2", n * H * es, act, (n, H)),
             ("act", n * F * es, act, (n, F)), ("head", n * H * es, act, (n, H)),
             ("fmods", 2 * 2 * H * 4, torch.float32, (2, 2 * H)), ("sched", 16, torch.int32, (4,))]
    out, off = {}, 0
    raw = ws.view(torch.uint8)
    for name, nbytes, dt, shape in sizes:
        out[name] = raw[off:off + nbytes].view(dt).view(shape)
        off += a256(nbytes)
    return out
