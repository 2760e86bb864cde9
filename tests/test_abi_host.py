"""CPU-side checks of the C ABI library: it loads, exports every entry point
that include/mmh3.h declares, and its host helpers (layouts, the flow-clock
remap, the timestep plan) agree exactly with the oracle.  No GPU compute."""

import ctypes as C
import glob
import os
import re

import numpy as np
import pytest
import torch

from oracle import mmh3_oracle as O
from packed_multimodal_diffusion_b200 import _lib, api, configs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:mmh3_status|double|void|int|long long|const char\s*\*)\s*(mmh3_\w+)\s*\(",
                             text, flags=re.M):
            names.add(m.group(1))
    return names


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    names = declared_symbols()
    assert len(names) >= 19
    for n in names:
        assert hasattr(lib, n), n
    assert set(_lib.SIGNATURES) == names
    assert lib.mmh3_version().startswith(b"mmh3-b200")
    # the boundary's calls under the names the design fixes
    for n in ("mmh3_time_shift_sigma", "mmh3_workspace_size", "mmh3_prepare_block_weights",
              "mmh3_resolve_rows", "mmh3_adaln_modulation", "mmh3_block_forward", "mmh3_stack_forward",
              "mmh3_vit_layer_forward", "mmh3_status_sync", "mmh3_last_error", "mmh3_layout_t2va",
              "mmh3_layout_image"):
        assert n in names, n


def test_time_shift_matches_oracle():
    for s in (1e-3, 0.1, 0.3, 0.5, 0.972973, 1.0):
        for (f, t) in ((12.0, 3.0), (3.0, 12.0)):
            assert api.time_shift_sigma(s, f, t) == O.time_shift_sigma(s, f, t)


@pytest.mark.parametrize("name", ["tiny", "block", "stack", "image"])
def test_layouts_bit_exact_against_oracle(name):
    c = configs.CONFIGS[name]
    if c.image_mode:
        segs, pos = api.layout_image(c.text_len, c.ref_lat_h, c.ref_lat_w, c.lat_h, c.lat_w)
        L = O.layout_image(c.text_len, c.ref_lat_h, c.ref_lat_w, c.lat_h, c.lat_w)
    else:
        segs, pos = api.layout_t2va(c.text_len, c.latent_t, c.lat_h, c.lat_w, c.audio_t)
        L = O.layout_t2va(c.text_len, c.latent_t, c.lat_h, c.lat_w, c.audio_t)
    assert [tuple(s) for s in segs] == [tuple(s) for s in L["segments"]]
    np.testing.assert_array_equal(pos, L["pos"].astype(np.float32))


def test_printed_t2va_layout_through_the_abi():
    segs, pos = api.layout_t2va(8, 3, 8, 12, 5)
    assert pos.shape == (90, 3)
    assert [s[2] for s in segs] == [1, 2, 0]


@pytest.mark.parametrize("sigma_v", [1e-9, 0.05, 0.3, 0.5, 0.9, 1.0])
@pytest.mark.parametrize("name", ["tiny", "image"])
def test_plan_timesteps_matches_oracle(name, sigma_v):
    c = configs.CONFIGS[name]
    if c.image_mode:
        L = O.layout_image(c.text_len, c.ref_lat_h, c.ref_lat_w, c.lat_h, c.lat_w)
    else:
        L = O.layout_t2va(c.text_len, c.latent_t, c.lat_h, c.lat_w, c.audio_t)
    sa = O.time_shift_sigma(max(sigma_v, 1e-6), 12, 3)
    ts_o, slot = O.plan_timesteps(sigma_v, sa, L["segments"])
    ts, rows = api.plan_timesteps(L["segments"], L["seq_len"], sigma_v, sa)
    assert ts == ts_o
    rows_o = O.token_rows(L["segments"], slot, L["seq_len"])
    for (a, b, _, _), r in zip(L["segments"], rows):
        assert (rows_o[a:b] == r).all()


def test_argument_errors_are_reported_before_launch():
    lib = _lib.load()
    d = api.make_dims(2688, 21, 128, 10752)
    bad = api.make_dims(2688, 21, 96, 10752)
    v = C.c_size_t()
    assert lib.mmh3_workspace_size(C.byref(bad), 100, C.byref(v)) == 2
    assert b"head_dim" in lib.mmh3_last_error()
    assert lib.mmh3_workspace_size(C.byref(d), 100, C.byref(v)) == 0 and v.value > 0
    # a block call with a null weight struct fails with MMH3_ERR_ARG, no CUDA involved
    segs = api.segments([(0, 10, 1, 0)])
    ws = C.c_void_p(256)  # never dereferenced: validation fails first
    rc = lib.mmh3_block_forward(C.byref(d), None, C.c_void_p(256), 10, segs, 1, None, 0.5, 0.2, 1,
                                None, ws, v.value, None)
    assert rc in (1, 4)
    # segments with a gap
    with pytest.raises(_lib.Mmh3Error) as e:
        api.plan_timesteps([(0, 4, 1, 0), (5, 9, 0, 0)], 9, 0.5, 0.2)
    assert e.value.code == 2


def test_host_fault_injection(monkeypatch):
    monkeypatch.setenv("MMH3_FAULT", "plan")
    with pytest.raises(_lib.Mmh3Error) as e:
        api.plan_timesteps([(0, 4, 1, 0)], 4, 0.5, 0.2)
    assert "injected fault at plan" in str(e.value)
    monkeypatch.delenv("MMH3_FAULT")
    ts, rows = api.plan_timesteps([(0, 4, 1, 0)], 4, 0.5, 0.2)
    assert ts == [0.5] and rows == [1]


def test_refine_and_embed_argument_checks():
    lib = _lib.load()
    d = api.make_dims(256, 2, 128, 512)
    v = C.c_size_t()
    # refiner workspace = block workspace + the fp32 residual stream, 256-byte aligned
    assert lib.mmh3_workspace_size(C.byref(d), 77, C.byref(v)) == 0
    blk = v.value
    assert api.refine_workspace_size(d, 77) == blk + ((77 * 256 * 4 + 255) // 256) * 256
    # patch rows staged in the act dtype: video rows T*(h/2)*(w/2) of 4C, audio rows 2T of C
    assert api.patch_embed_workspace_size(d, api.MMH3_STREAM_VIDEO, (16, 3, 10, 14)) == \
        ((3 * 5 * 7 * 64 * 2 + 255) // 256) * 256
    assert api.patch_embed_workspace_size(d, api.MMH3_STREAM_AUDIO, (24, 2, 37)) == \
        ((74 * 24 * 2 + 255) // 256) * 256
    assert lib.mmh3_patch_embed_workspace_size(C.byref(d), 0, 4, 1, 3, 4, C.byref(v)) == 2
    assert lib.mmh3_patch_embed_workspace_size(C.byref(d), 1, 4, 1, 2, 4, C.byref(v)) == 1
    # K * 2 bytes = 6 is not a multiple of 16: rejected before any launch
    rc = lib.mmh3_patch_embed(C.byref(d), 2, C.c_void_p(256), 3, 4, 0, 0, C.c_void_p(256),
                              C.c_void_p(256), C.c_void_p(256), C.c_void_p(256), 1 << 20, None)
    assert rc == 2 and b"K = 3" in lib.mmh3_last_error()
    # embed: segment rows must match the streams; condition frames must match the segments
    L = O.layout_t2va(5, 2, 6, 8, 7)
    segs = api.segments(L["segments"])
    fake = C.c_void_p(256)
    ew = _lib.EmbedWeights(fake, fake, fake, fake)

    def inputs(frames, n_cond=0):
        return _lib.EmbedInputs(fake, fake, 4, frames, 6, 8, fake, 8, 7, None, n_cond)

    rc = lib.mmh3_embed(C.byref(d), segs, 3, L["seq_len"], C.byref(inputs(3)), C.byref(ew), fake,
                        fake, 1 << 20, None)
    assert rc == 2 and b"video segment" in lib.mmh3_last_error()
    rc = lib.mmh3_embed(C.byref(d), segs, 3, L["seq_len"], C.byref(inputs(2, 1)), C.byref(ew),
                        fake, fake, 1 << 20, None)
    assert rc == 1 and b"condition frames" in lib.mmh3_last_error()


def test_new_entry_points_reject_bad_arguments_before_launch():
    lib = _lib.load()
    d = api.make_dims(256, 2, 128, 512)
    fake = C.c_void_p(256)
    segs = api.segments([(0, 10, 1, 0)])
    # host-buffer block: slot in [0, HOST_SLOTS); pos_host / pos_dev both or neither
    for bad in (-1, api.HOST_SLOTS):
        rc = lib.mmh3_block_forward_host(C.byref(d), None, fake, fake, 10, segs, 1, fake, 0.5, 0.2, bad, fake,
                                         fake, fake, 1 << 20, None, None, None)
        assert rc == 1 and b"slot" in lib.mmh3_last_error()
    rc = lib.mmh3_block_forward_host(C.byref(d), None, fake, fake, 10, segs, 1, fake, 0.5, 0.2, 0, fake,
                                     None, fake, 1 << 20, None, None, None)
    assert rc == 1 and b"pos_host" in lib.mmh3_last_error()
    # shard block: fp32 activations are not supported; kv pointers are required
    d32 = api.make_dims(256, 4, 64, 512, act_dtype=torch.float32)
    v = C.c_size_t()
    lib.mmh3_workspace_size(C.byref(d32), 10, C.byref(v))
    rc = lib.mmh3_block_cp_begin(C.byref(d32), None, fake, 10, segs, 1, None, 0.5, 0.2, 1, fake, fake,
                                 v.value, None)
    assert rc == 5
    lib.mmh3_workspace_size(C.byref(d), 10, C.byref(v))
    rc = lib.mmh3_block_cp_end(C.byref(d), None, fake, 10, segs, 1, 0.5, 0.2, 1, None, 10, fake, v.value,
                               None)
    assert rc == 1 and b"kv_all" in lib.mmh3_last_error()
    rc = lib.mmh3_block_cp_end(C.byref(d), None, fake, 10, segs, 1, 0.5, 0.2, 1, fake, 9, fake, v.value,
                               None)
    assert rc == 2 and b"n_kv" in lib.mmh3_last_error()
    # refiner: text_dim * 2 bytes must be a multiple of 16
    lib.mmh3_refine_workspace_size(C.byref(d), 10, C.byref(v))
    rc = lib.mmh3_refine_text(C.byref(d), fake, 10, 12, fake, fake, None, 0, fake, 1e-6, fake, fake, v.value,
                              None)
    assert rc == 2 and b"text_dim" in lib.mmh3_last_error()
    # forward: the video head width must be 4 x the latent channels
    L = O.layout_t2va(5, 2, 6, 8, 7)
    fsegs = api.segments(L["segments"])
    ins = _lib.EmbedInputs(fake, fake, 4, 2, 6, 8, fake, 8, 7, None, 0)
    ew = _lib.EmbedWeights(fake, fake, fake, fake)
    hw = _lib.HeadWeights(fake, fake, fake, fake, fake, fake, fake, fake, 32, 8)
    lib.mmh3_forward_workspace_size(C.byref(d), L["seq_len"], C.byref(ins), C.byref(v))
    rc = lib.mmh3_forward(C.byref(d), fsegs, 3, L["seq_len"], None, 0.5, 0.2, C.byref(ins), C.byref(ew), None, 0,
                          C.byref(hw), fake, fake, fake, fake, v.value, None)
    assert rc == 2 and b"video head width" in lib.mmh3_last_error()
    # the launch counter exists and never goes backwards
    assert lib.mmh3_launch_count() >= 0


def test_host_slot_count_matches_header():
    text = open(os.path.join(ROOT, "include", "mmh3.h")).read()
    m = re.search(r"#define MMH3_HOST_SLOTS (\d+)", text)
    assert m and int(m.group(1)) == api.HOST_SLOTS


# ---------------------------------------------- keyframe / reference layouts
FL2VA_CASES = [
    ((8, 3, 8, 12, 5), [(0, 39), (38, 39)], None),
    ((20, 3, 16, 20, 20), [(38, 39)], [1] * 5 + [0] * 10 + [1] * 5),
    ((16, 2, 8, 8, 8), [], None),
]
REF2VA_CASES = [
    ((4, 2, 4, 4, 3), [("image", 4, 6)], None),
    ((4, 2, 4, 4, 3), [("audio", 3)], None),
    ((4, 2, 4, 4, 3), [("video", 2, 4, 8, 5)], None),
    ((10, 3, 16, 20, 6), [("image", 8, 8), ("audio", 4), ("video", 3, 8, 12, 0), ("video", 1, 4, 4, 7)],
     [1, 1, 1, 0, 0, 0, 0, 1, 1, 1]),
]


@pytest.mark.parametrize("case", range(len(FL2VA_CASES)))
def test_fl2va_layout_bit_exact_against_oracle(case):
    sizes, frames, tags = FL2VA_CASES[case]
    segs, pos = api.layout_fl2va(*sizes, frames, tags)
    L = O.layout_fl2va(*sizes, frames, text_tags=tags)
    assert [tuple(s) for s in segs] == [tuple(s) for s in L["segments"]]
    np.testing.assert_array_equal(pos, L["pos"].astype(np.float32))


@pytest.mark.parametrize("case", range(len(REF2VA_CASES)))
def test_ref2va_layout_bit_exact_against_oracle(case):
    sizes, refs, tags = REF2VA_CASES[case]
    segs, pos = api.layout_ref2va(*sizes, refs, tags)
    L = O.layout_ref2va(*sizes, refs, text_tags=tags)
    assert [tuple(s) for s in segs] == [tuple(s) for s in L["segments"]]
    np.testing.assert_array_equal(pos, L["pos"].astype(np.float32))


@pytest.mark.parametrize("sigma_v", [1e-9, 1e-4, 0.3, 0.9, 1.0])
def test_condition_clock_plan_matches_oracle(sigma_v):
    sa = O.time_shift_sigma(max(sigma_v, 1e-6), 12, 3)
    for L in (O.layout_fl2va(*FL2VA_CASES[0][0], FL2VA_CASES[0][1]),
              O.layout_ref2va(*REF2VA_CASES[3][0], REF2VA_CASES[3][1], text_tags=REF2VA_CASES[3][2])):
        ts_o, slot = O.plan_timesteps(sigma_v, sa, L["segments"])
        ts, rows = api.plan_timesteps(L["segments"], L["seq_len"], sigma_v, sa)
        assert ts == ts_o
        rows_o = O.token_rows(L["segments"], slot, L["seq_len"])
        assert [int(rows_o[a]) for a, _, _, _ in L["segments"]] == rows


def test_layout_errors_and_more_than_two_timesteps_without_modulation():
    lib = _lib.load()
    kf = (_lib.Keyframe * 1)(_lib.Keyframe(5, 39))
    segs = (_lib.Segment * 16)()
    ns, n = C.c_int(), C.c_int()
    # a keyframe that is neither the first nor the last frame
    assert lib.mmh3_layout_fl2va(8, 3, 8, 12, 5, kf, 1, None, segs, 16, C.byref(ns), None, 0, C.byref(n)) == 1
    assert b"first and the last" in lib.mmh3_last_error() or b"first and last" in lib.mmh3_last_error()
    # segment capacity below the layout's count
    kf2 = (_lib.Keyframe * 2)(_lib.Keyframe(0, 39), _lib.Keyframe(38, 39))
    assert lib.mmh3_layout_fl2va(8, 3, 8, 12, 5, kf2, 2, None, segs, 4, C.byref(ns), None, 0, C.byref(n)) == 2
    # four distinct timesteps: the block's own adaLN curve is refused before
    # any launch (nothing below is dereferenced)
    sizes, refs, tags = REF2VA_CASES[3]
    L = O.layout_ref2va(*sizes, refs, text_tags=tags)
    nn = L["seq_len"]
    d = api.make_dims(256, 2, 128, 512)
    v = C.c_size_t()
    assert lib.mmh3_workspace_size(C.byref(d), nn, C.byref(v)) == 0
    w = _lib.BlockWeights(*([256] * 11))
    sa = O.time_shift_sigma(0.3, 12, 3)
    rc = lib.mmh3_block_forward(C.byref(d), C.byref(w), C.c_void_p(256), nn, api.segments(L["segments"]),
                                len(L["segments"]), None, 0.3, sa, 1, None, C.c_void_p(256), v.value, None)
    assert rc == 5 and b"two slots" in lib.mmh3_last_error()
    out = C.c_int()
    rc = lib.mmh3_adaln_modulation(C.byref(d), C.c_void_p(256), C.c_void_p(256), C.c_void_p(256), 18 * 256,
                                   api.segments(L["segments"]), len(L["segments"]), nn, 0.3, sa,
                                   C.c_void_p(256), C.byref(out), None)
    assert rc == 5 and out.value == 4


def test_check_mode_canaries_enlarge_the_workspace_and_clock_validation():
    d = api.make_dims(256, 2, 128, 512)
    base = api.workspace_size(d, 300)
    try:
        api.set_check(1)
        assert _lib.load().mmh3_check_enabled() == 1
        # ten regions (the last one attention's work counter), a 256-byte
        # canary after each
        assert api.workspace_size(d, 300) == base + 10 * 256
    finally:
        api.set_check(-1)
    assert api.workspace_size(d, 300) == base
    # a forged clock outside the four is refused by the host before any launch
    with pytest.raises(_lib.Mmh3Error) as e:
        api.plan_timesteps([(0, 4, 1, 0), (4, 9, 0, 7)], 9, 0.5, 0.2)
    assert e.value.code == 1 and "clock 7" in str(e.value)


def test_workspace_fault_injection_before_any_launch(monkeypatch):
    lib = _lib.load()
    d = api.make_dims(256, 2, 128, 512)
    v = C.c_size_t()
    assert lib.mmh3_workspace_size(C.byref(d), 300, C.byref(v)) == 0
    w = _lib.BlockWeights(*([256] * 11))
    segs = api.segments([(0, 300, 1, 0)])
    monkeypatch.setenv("MMH3_FAULT", "workspace")
    rc = lib.mmh3_block_forward(C.byref(d), C.byref(w), C.c_void_p(256), 300, segs, 1, None, 0.5, 0.2, 1, None,
                                C.c_void_p(256), v.value, None)
    assert rc == 4 and b"injected fault at workspace" in lib.mmh3_last_error()
