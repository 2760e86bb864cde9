"""ctypes declarations of the C ABI in include/mmh3.h (argument marshalling
only).  Loading fails loudly when libmmh3.so is missing: there is no CPU or
Python fallback for any step of the path."""

from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmmh3.so")

MMH3_F32, MMH3_BF16 = 0, 1

STATUS_NAMES = {0: "MMH3_OK", 1: "MMH3_ERR_ARG", 2: "MMH3_ERR_SHAPE", 3: "MMH3_ERR_ALIGN",
                4: "MMH3_ERR_WORKSPACE", 5: "MMH3_ERR_UNSUPPORTED", 6: "MMH3_ERR_CUDA",
                7: "MMH3_ERR_TIMEOUT", 8: "MMH3_ERR_CHECK"}


class Mmh3Error(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


class Dims(C.Structure):
    _fields_ = [("hidden", C.c_int), ("heads", C.c_int), ("head_dim", C.c_int), ("ffn", C.c_int),
                ("rank", C.c_int), ("grid", C.c_int), ("rope_k", C.c_int), ("eps", C.c_float),
                ("qk_eps", C.c_float), ("rope_theta", C.c_float), ("act_dtype", C.c_int)]


class Segment(C.Structure):
    _fields_ = [("start", C.c_uint32), ("stop", C.c_uint32), ("tag", C.c_uint8),
                ("clock", C.c_uint8), ("pad", C.c_uint8 * 2)]


class Keyframe(C.Structure):
    _fields_ = [("pixel_index", C.c_int), ("frame_count", C.c_int)]


class Ref(C.Structure):
    _fields_ = [("kind", C.c_int), ("lat_h", C.c_int), ("lat_w", C.c_int), ("latent_t", C.c_int),
                ("audio_t", C.c_int)]


MMH3_REF_IMAGE, MMH3_REF_AUDIO, MMH3_REF_VIDEO = 0, 1, 2


class BlockWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("norm1", "norm2", "wqkv", "wout", "q_norm", "k_norm",
                                          "wfc1", "wfc2", "adaln_w", "adaln_b", "adaln_table")]


class HeadWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("final_norm", "adaln_w", "adaln_b", "adaln_table",
                                          "w_video", "b_video", "w_audio", "b_audio")] + \
               [("out_video", C.c_int), ("out_audio", C.c_int)]


class VitDims(C.Structure):
    _fields_ = [("hidden", C.c_int), ("heads", C.c_int), ("head_dim", C.c_int), ("mlp", C.c_int),
                ("ln_eps", C.c_float)]


class VitWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("ln1_g", "ln1_b", "wqkv", "bqkv", "wo", "bo", "ln2_g",
                                          "ln2_b", "w1", "b1", "w2", "b2")]


class EmbedInputs(C.Structure):
    _fields_ = [("text", C.c_void_p), ("video", C.c_void_p), ("video_channels", C.c_int),
                ("video_frames", C.c_int), ("lat_h", C.c_int), ("lat_w", C.c_int),
                ("audio", C.c_void_p), ("audio_channels", C.c_int), ("audio_frames", C.c_int),
                ("cond", C.POINTER(C.c_void_p)), ("n_cond", C.c_int)]


class EmbedWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("w_video", "b_video", "w_audio", "b_audio")]


MMH3_STREAM_VIDEO, MMH3_STREAM_AUDIO = 0, 2

_P = C.c_void_p
_I = C.c_int
_D = C.c_double
_SEGP = C.POINTER(Segment)

# name -> (restype, argtypes)
SIGNATURES = {
    "mmh3_time_shift_sigma": (C.c_double, [_D, _D, _D]),
    "mmh3_layout_t2va": (_I, [_I, _I, _I, _I, _I, _SEGP, C.POINTER(_I), C.POINTER(C.c_float), _I,
                              C.POINTER(_I)]),
    "mmh3_layout_image": (_I, [_I, _I, _I, _I, _I, _SEGP, C.POINTER(_I), C.POINTER(C.c_float), _I,
                               C.POINTER(_I)]),
    "mmh3_layout_fl2va": (_I, [_I, _I, _I, _I, _I, C.POINTER(Keyframe), _I, C.POINTER(C.c_uint8), _SEGP, _I,
                               C.POINTER(_I), C.POINTER(C.c_float), _I, C.POINTER(_I)]),
    "mmh3_layout_ref2va": (_I, [_I, _I, _I, _I, _I, C.POINTER(Ref), _I, C.POINTER(C.c_uint8), _SEGP, _I,
                                C.POINTER(_I), C.POINTER(C.c_float), _I, C.POINTER(_I)]),
    "mmh3_plan_timesteps": (_I, [_SEGP, _I, _I, _D, _D, C.POINTER(_D), C.POINTER(_I),
                                 C.POINTER(_I)]),
    "mmh3_resolve_rows": (_I, [_SEGP, _I, _I, _D, _D, _P, _P]),
    "mmh3_adaln_modulation": (_I, [C.POINTER(Dims), _P, _P, _P, _I, _SEGP, _I, _I, _D, _D, _P,
                                   C.POINTER(_I), _P]),
    "mmh3_prepare_block_weights": (_I, [C.POINTER(Dims), _P, _P, _P]),
    "mmh3_prepare_fc1": (_I, [C.POINTER(Dims), _P, _P, _P]),
    "mmh3_workspace_size": (_I, [C.POINTER(Dims), _I, C.POINTER(C.c_size_t)]),
    "mmh3_attention": (_I, [_P, _I, _I, _I, _I, _I, C.c_float, _P, _P]),
    "mmh3_attention_ws": (_I, [_P, _I, _I, _I, _I, _I, C.c_float, _P, _P, C.c_size_t, _P]),
    "mmh3_block_forward": (_I, [C.POINTER(Dims), C.POINTER(BlockWeights), _P, _I, _SEGP, _I, _P,
                                _D, _D, _I, _P, _P, C.c_size_t, _P]),
    "mmh3_block_forward_noalloc": (_I, [C.POINTER(Dims), C.POINTER(BlockWeights), _P, _I, _SEGP, _I,
                                        _P, _D, _D, _I, _P]),
    "mmh3_stack_forward": (_I, [C.POINTER(Dims), C.POINTER(BlockWeights), _I,
                                C.POINTER(HeadWeights), _P, _I, _SEGP, _I, _P, _D, _D, _P, _P, _P,
                                C.c_size_t, _P]),
    "mmh3_block_forward_host": (_I, [C.POINTER(Dims), C.POINTER(BlockWeights), _P, _P, _I, _SEGP, _I,
                                     _P, _D, _D, _I, _P, _P, _P, C.c_size_t, _P, _P, _P]),
    "mmh3_block_cp_begin": (_I, [C.POINTER(Dims), C.POINTER(BlockWeights), _P, _I, _SEGP, _I, _P,
                                 _D, _D, _I, _P, _P, C.c_size_t, _P]),
    "mmh3_block_cp_end": (_I, [C.POINTER(Dims), C.POINTER(BlockWeights), _P, _I, _SEGP, _I, _D, _D,
                               _I, _P, _I, _P, C.c_size_t, _P]),
    "mmh3_refine_workspace_size": (_I, [C.POINTER(Dims), _I, C.POINTER(C.c_size_t)]),
    "mmh3_refine_text": (_I, [C.POINTER(Dims), _P, _I, _I, _P, _P, C.POINTER(BlockWeights), _I, _P,
                              C.c_float, _P, _P, C.c_size_t, _P]),
    "mmh3_patch_embed_workspace_size": (_I, [C.POINTER(Dims), _I, _I, _I, _I, _I,
                                             C.POINTER(C.c_size_t)]),
    "mmh3_patch_embed": (_I, [C.POINTER(Dims), _I, _P, _I, _I, _I, _I, _P, _P, _P, _P, C.c_size_t,
                              _P]),
    "mmh3_embed_workspace_size": (_I, [C.POINTER(Dims), C.POINTER(EmbedInputs),
                                       C.POINTER(C.c_size_t)]),
    "mmh3_embed": (_I, [C.POINTER(Dims), _SEGP, _I, _I, C.POINTER(EmbedInputs),
                        C.POINTER(EmbedWeights), _P, _P, C.c_size_t, _P]),
    "mmh3_forward_workspace_size": (_I, [C.POINTER(Dims), _I, C.POINTER(EmbedInputs),
                                         C.POINTER(C.c_size_t)]),
    "mmh3_forward": (_I, [C.POINTER(Dims), _SEGP, _I, _I, _P, _D, _D, C.POINTER(EmbedInputs),
                          C.POINTER(EmbedWeights), C.POINTER(BlockWeights), _I,
                          C.POINTER(HeadWeights), _P, _P, _P, _P, C.c_size_t, _P]),
    "mmh3_unpatchify_video": (_I, [_P, _I, _I, _I, _I, _P, _P]),
    "mmh3_unpack_audio": (_I, [_P, _I, _I, _P, _P]),
    "mmh3_vit_fold_qkv": (_I, [C.POINTER(VitDims), _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "mmh3_vit_workspace_size": (_I, [C.POINTER(VitDims), _I, _I, C.POINTER(C.c_size_t)]),
    "mmh3_vit_layer_forward": (_I, [C.POINTER(VitDims), C.POINTER(VitWeights), _P, _I, _I, _P,
                                    C.c_size_t, _P]),
    "mmh3_device_status": (_I, [_P, C.POINTER(_I), C.POINTER(_I)]),
    "mmh3_status_sync": (_I, [_P, C.POINTER(_I)]),
    "mmh3_set_wait_limit_ns": (None, [C.c_uint64]),
    "mmh3_set_check": (None, [_I]),
    "mmh3_check_enabled": (_I, []),
    "mmh3_selftest_wait_timeout": (_I, [C.c_uint64, _P]),
    "mmh3_prof_enable": (None, [_I]),
    "mmh3_prof_collect": (_I, [C.POINTER(C.c_double), _I, C.POINTER(C.c_long)]),
    "mmh3_prof_reset": (None, []),
    "mmh3_prof_collect_kernels": (_I, [C.POINTER(C.c_double), C.POINTER(C.c_long), _I]),
    "mmh3_last_error": (C.c_char_p, []),
    "mmh3_launch_count": (C.c_longlong, []),
    "mmh3_version": (C.c_char_p, []),
}

_lib = None


def load() -> C.CDLL:
    """Load libmmh3.so (built by ``build.py``); raise if it is absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m packed_multimodal_diffusion_b200.build` (no fallback exists)")
    lib = C.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def check(code: int) -> None:
    if code != 0:
        msg = load().mmh3_last_error().decode(errors="replace")
        raise Mmh3Error(code, msg)
