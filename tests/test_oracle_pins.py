"""Pins for the CPU oracle: checks against what the pages and the mathematics
fix, never against the oracle's own formulas retyped.

Sources: "cortiq_engine/mmh3.rs" (cortiq-engine 0.5.72) -- its own unit tests
and doc comments; "ffai-argus 0.7.0 src/siglip.rs" -- its GELU landmarks;
textbook identities (rotation matrices, softmax, LayerNorm moments).
"""

import json
import math
import os
import random

import numpy as np
import pytest
import torch

from oracle import mmh3_oracle as O
from packed_multimodal_diffusion_b200 import configs, synth

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                   "mmh3_printed_values.json")))


# ---------------------------------------------------------------- schedule

def test_remap_involution_printed_points():
    g = GOLD["schedule_remap_is_an_involution"]
    for s in g["sigmas"]:
        a = O.time_shift_sigma(s, g["from_shift"], g["to_shift"])
        back = O.time_shift_sigma(a, g["to_shift"], g["from_shift"])
        assert abs(back - s) < g["tol"]


def test_remap_closed_form_12_to_3():
    # base = s/(12 - 11 s); 3b/(1 + 2b) simplifies to s/(4 - 3 s).
    for s in np.linspace(0.0, 1.0, 101):
        assert O.time_shift_sigma(s, 12.0, 3.0) == pytest.approx(s / (4 - 3 * s), abs=1e-15)
    # tiny workload: t_v = 0.7 -> sigma_a = 3/31, t_a = 28/31
    assert O.time_shift_sigma(0.3, 12.0, 3.0) == pytest.approx(3.0 / 31.0, abs=1e-15)


def test_slope_matches_finite_difference_printed_points():
    g = GOLD["slope_matches_a_finite_difference"]
    h = g["h"]
    for s in g["sigmas"]:
        num = (O.time_shift_sigma(s + h, 12, 3) - O.time_shift_sigma(s - h, 12, 3)) / (2 * h)
        assert abs(num - O.time_shift_slope(s, 12, 3)) < g["tol"]
    # closed form of the derivative of s/(4-3s): 4/(4-3s)^2
    for s in (0.1, 0.4, 0.7):
        assert O.time_shift_slope(s, 12, 3) == pytest.approx(4 / (4 - 3 * s) ** 2, rel=1e-12)


# ------------------------------------------------------------------ layout

def test_axis_from_sqrt_area_is_the_documented_linspace():
    # doc comment: linspace((1-ratio)/2, (1+ratio)/2, dim/patch, endpoint=False) * 32
    for (h, w) in ((8, 12), (60, 104), (128, 128), (8, 8)):
        area = math.sqrt(h * w)
        for dim in (h, w):
            r = dim / area
            ref = np.linspace((1 - r) / 2, (1 + r) / 2, dim // 2, endpoint=False) * 32
            np.testing.assert_allclose(O.axis_from_sqrt_area(dim, 2, area), ref,
                                       rtol=0, atol=1e-12)


def test_t2va_printed_layout():
    g = GOLD["layout_places_the_target_streams_last"]
    a = g["args"]
    L = O.layout_t2va(a["text_len"], a["latent_t"], a["lat_h"], a["lat_w"], a["audio_t"])
    assert L["frame_rows"] == g["frame_rows"]
    assert L["seq_len"] == g["seq_len"] == L["pos"].shape[0]
    tags = [s[2] for s in L["segments"]]
    assert tags == [O.TAG_TEXT, O.TAG_AUDIO, O.TAG_VIDEO]
    v0 = L["segments"][2][0]
    t0 = L["pos"][v0, 0]
    t1 = L["pos"][v0 + L["frame_rows"], 0]
    assert abs(t1 - t0 - g["video_dt_frame0_to_frame1"]) < g["tol"]
    # second span of the [1,4,4,4,4] pattern: 4 * 5/3
    t2 = L["pos"][v0 + 2 * L["frame_rows"], 0]
    assert abs(t2 - t1 - 4 * GOLD["frame_per_token"]["rescale"]) < 1e-12


def test_t2va_text_and_audio_positions():
    L = O.layout_t2va(8, 3, 8, 12, 5)
    pos = L["pos"]
    # text rows [i, 0, 0]
    np.testing.assert_array_equal(pos[:8], np.stack([np.arange(8), np.zeros(8), np.zeros(8)], 1))
    # audio: two channels of 5 frames from the text's end; h = 0; w at the
    # frame grid's extremes (low for channel 0, high for channel 1)
    w_axis = np.linspace((1 - 12 / math.sqrt(96)) / 2, (1 + 12 / math.sqrt(96)) / 2, 6,
                         endpoint=False) * 32
    a = pos[8:18]
    np.testing.assert_allclose(a[:5, 0], 8 + np.arange(5))
    np.testing.assert_allclose(a[5:, 0], 8 + np.arange(5))
    assert (a[:, 1] == 0).all()
    np.testing.assert_allclose(a[:5, 2], w_axis[0], atol=1e-12)
    np.testing.assert_allclose(a[5:, 2], w_axis[-1], atol=1e-12)
    # video starts at the same origin as audio
    assert pos[18, 0] == 8.0


@pytest.mark.parametrize("name,n", [("tiny", 64), ("block", 13248), ("stack", 26496),
                                    ("image", 8448)])
def test_workload_sequence_lengths(name, n):
    c = configs.CONFIGS[name]
    if c.image_mode:
        L = O.layout_image(c.text_len, c.ref_lat_h, c.ref_lat_w, c.lat_h, c.lat_w)
    else:
        L = O.layout_t2va(c.text_len, c.latent_t, c.lat_h, c.lat_w, c.audio_t)
    assert L["seq_len"] == n == c.seq_len


def test_image_layout_reading():
    L = O.layout_image(4, 4, 4, 4, 4)
    pos = L["pos"]
    assert L["seq_len"] == 4 + 4 + 4
    assert [s[2] for s in L["segments"]] == [O.TAG_TEXT, O.TAG_VIDEO, O.TAG_VIDEO]
    assert (pos[4:8, 0] == 4).all() and (pos[8:12, 0] == 5).all()
    # square grid: 32 i / n
    np.testing.assert_allclose(sorted(set(pos[4:8, 1])), [0.0, 16.0])


# --------------------------------------------------------------------- rows

def _rows(name, sigma_v):
    c = configs.CONFIGS[name]
    if c.image_mode:
        L = O.layout_image(c.text_len, c.ref_lat_h, c.ref_lat_w, c.lat_h, c.lat_w)
    else:
        L = O.layout_t2va(c.text_len, c.latent_t, c.lat_h, c.lat_w, c.audio_t)
    sa = O.time_shift_sigma(max(sigma_v, 1e-6), 12, 3)
    ts, slot = O.plan_timesteps(sigma_v, sa, L["segments"])
    return ts, O.token_rows(L["segments"], slot, L["seq_len"]), L


def test_rows_two_clocks_hand_enumerated():
    ts, rows, L = _rows("block", 0.5)
    # t_v = 0.5, sigma_a = 0.5/2.5 = 0.2 -> t_a = 0.8 > t_v: video slot 0, audio slot 1
    assert ts == pytest.approx([0.5, 0.8])
    assert rows[:256].tolist() == [1] * 256            # text: slot 0, tag 1
    assert rows[256:768].tolist() == [5] * 512         # audio: slot 1, tag 2
    assert set(rows[768:].tolist()) == {0}             # video: slot 0, tag 0
    ts, rows, _ = _rows("tiny", 0.3)
    assert ts == pytest.approx([0.7, 28 / 31])
    assert sorted(set(rows.tolist())) == [0, 1, 5]


def test_rows_tied_clocks_and_image_mode():
    ts, rows, _ = _rows("tiny", 1.0)        # sigma_v = 1 -> t_v = t_a = 0
    assert ts == [0.0] and sorted(set(rows.tolist())) == [0, 1, 2]
    ts, rows, _ = _rows("image", 0.5)
    assert len(ts) == 1 and sorted(set(rows.tolist())) == [0, 1]
    assert (rows[:256] == 1).all() and (rows[256:] == 0).all()


# ------------------------------------------------------------------- adaLN

def test_adaln_exact_at_nodes_and_clamped():
    table = np.random.default_rng(0).standard_normal((1025, 24))
    for i in (0, 1, 511, 1023, 1024):
        np.testing.assert_array_equal(O.adaln_coords(table, i / 1024), table[i])
    np.testing.assert_array_equal(O.adaln_coords(table, -3.0), table[0])
    np.testing.assert_array_equal(O.adaln_coords(table, 7.0), table[1024])


def test_adaln_linear_between_nodes():
    table = np.random.default_rng(1).standard_normal((1025, 24))
    for i in (0, 100, 1023):
        mid = O.adaln_coords(table, (i + 0.5) / 1024)
        np.testing.assert_allclose(mid, 0.5 * (table[i] + table[i + 1]), atol=1e-13)
        q = O.adaln_coords(table, (i + 0.25) / 1024)
        np.testing.assert_allclose(q, 0.75 * table[i] + 0.25 * table[i + 1], atol=1e-13)


def test_adaln_zero_basis_gives_bias_and_one_hot_picks_coordinate():
    H, R = 4, 24
    rows_per_slot = 3 * 6 * H
    table = np.arange(1025 * R, dtype=np.float64).reshape(1025, R)
    b = np.random.default_rng(2).standard_normal(2 * rows_per_slot)
    ts = [256 / 1024, 768 / 1024]
    m = O.block_mods(np.zeros((2 * rows_per_slot, R)), b, table, ts, H)
    np.testing.assert_array_equal(m.reshape(-1), b)
    # one-hot rows: basis row r picks coordinate k of ITS slot's timestep
    w = np.zeros((2 * rows_per_slot, R))
    w[5, 3] = 1.0                       # slot 0 (video clock row block)
    w[rows_per_slot + 7, 11] = 1.0      # slot 1
    m = O.block_mods(w, np.zeros(2 * rows_per_slot), table, ts, H).reshape(-1)
    assert m[5] == table[256, 3]
    assert m[rows_per_slot + 7] == table[768, 11]
    assert np.count_nonzero(m) == 2
    # one timestep: only the first slot's rows are evaluated
    m1 = O.block_mods(w, np.zeros(2 * rows_per_slot), table, [0.5], H)
    assert m1.shape == (3, 6 * H) and m1.reshape(-1)[5] == table[512, 3]


def test_final_mods_one_hot_picks_its_slots_timestep():
    # Final layer: rows_per_slot = 2H (chunks shift, scale), row = slot.  A
    # one-hot basis row in slot 1 picks coordinate k of ts[1]; slot 0's rows
    # come from ts[0].  A swapped slot order or a transposed [T_s, 2H]
    # reshape moves the ones.
    H, R = 5, 24
    rps = 2 * H
    table = np.arange(1025 * R, dtype=np.float64).reshape(1025, R) * 0.5
    ts = [128 / 1024, 896 / 1024]
    w = np.zeros((2 * rps, R))
    w[3, 7] = 1.0              # slot 0, shift chunk, element 3
    w[rps + H + 1, 19] = 1.0   # slot 1, scale chunk, element 1
    fm = O.final_mods(w, np.zeros(2 * rps), table, ts, H)
    assert fm.shape == (2, 2 * H)
    assert fm[0, 3] == table[128, 7]
    assert fm[1, H + 1] == table[896, 19]
    assert np.count_nonzero(fm) == 2
    # with a single timestep only slot 0 is evaluated
    fm1 = O.final_mods(w, np.zeros(2 * rps), table, [896 / 1024], H)
    assert fm1.shape == (1, 2 * H) and fm1[0, 3] == table[896, 7] and np.count_nonzero(fm1) == 1


def test_block_mods_row_and_chunk_addressing():
    # row = slot*3 + tag; chunk e of that row starts at e*H (modulate doc)
    H = 2
    rows_per_slot = 18 * H
    w = np.zeros((2 * rows_per_slot, 24))
    b = np.arange(2 * rows_per_slot, dtype=np.float64)
    m = O.block_mods(w, b, np.zeros((1025, 24)), [0.1, 0.9], H)
    assert m.shape == (6, 6 * H)
    # row 5 = slot 1, tag 2 (audio); chunk 2 (gate_msa)
    np.testing.assert_array_equal(O.chunk(m[5], 2, H), b[5 * 6 * H + 2 * H: 5 * 6 * H + 3 * H])


# --------------------------------------------------------- norms, modulate

def test_rms_norm_closed_forms():
    x = np.array([[3.0, 4.0]])
    np.testing.assert_allclose(O.rms_norm(x, np.ones(2), 0.0), [[3 / math.sqrt(12.5), 4 / math.sqrt(12.5)]])
    c = np.full((1, 16), -2.5)
    np.testing.assert_allclose(O.rms_norm(c, np.ones(16), 1e-5), -2.5 / math.sqrt(6.25 + 1e-5))
    g = np.linspace(0.5, 1.5, 16)
    np.testing.assert_allclose(O.rms_norm(c, g, 0.0)[0], -g)  # gain after the normalisation


def test_modulate_zero_is_identity():
    x = np.random.default_rng(3).standard_normal((5, 8))
    np.testing.assert_array_equal(O.modulate(x, np.zeros(8), np.zeros(8)), x)
    np.testing.assert_allclose(O.modulate(x, np.ones(8), np.ones(8)), 2 * x + 1)


def test_silu_and_gelu_landmarks():
    from scipy.special import erf, expit
    v = np.linspace(-8, 8, 33)
    np.testing.assert_allclose(O.silu(v), v * expit(v), rtol=1e-13)
    assert O.silu(np.array(0.0)) == 0.0
    # siglip.rs GELU landmarks
    assert abs(O.gelu_tanh(np.array(0.0))) < 1e-9
    assert abs(O.gelu_tanh(np.array(-10.0))) < 1e-6
    assert abs(O.gelu_tanh(np.array(10.0)) - 10.0) < 1e-4
    assert -0.18 < O.gelu_tanh(np.array(-0.75)) < -0.15
    # the tanh form tracks the exact erf GELU to within 1e-3 everywhere
    x = np.linspace(-6, 6, 2001)
    exact = 0.5 * x * (1 + erf(x / math.sqrt(2)))
    assert np.max(np.abs(O.gelu_tanh(x) - exact)) < 1e-3
    # monotone above its dip
    y = O.gelu_tanh(np.linspace(-0.7, 6, 500))
    assert (np.diff(y) > 0).all()


def test_layer_norm_moments():
    x = np.random.default_rng(4).standard_normal((7, 64)) * 3 + 5
    y = O.layer_norm(x, np.ones(64), np.zeros(64), 0.0)
    np.testing.assert_allclose(y.mean(-1), 0, atol=1e-12)
    np.testing.assert_allclose((y * y).mean(-1), 1, atol=1e-12)
    g, b = np.linspace(1, 2, 64), np.linspace(-1, 1, 64)
    np.testing.assert_allclose(O.layer_norm(x, g, b, 0.0), y * g + b, atol=1e-12)


# -------------------------------------------------------------------- rope

def test_rope_frequencies_match_the_per_axis_formulas():
    gr = GOLD["rope"]
    k = gr["per_axis"]
    assert k == gr["head_dim"] // 8 and 3 * k == gr["pairs"]
    f = O.rope_inv_freq(k, 10000.0)
    d = 2 * k                                       # 1-D rotate-half: theta^(-2j/d)
    np.testing.assert_allclose(f, np.power(10000.0, -2.0 * np.arange(k) / d), rtol=1e-15)
    np.testing.assert_allclose(f, np.exp(-math.log(10000.0) * np.arange(k) / k), rtol=1e-14)


def test_rope_rotates_unit_vector_by_the_right_angle_and_pair():
    hd, k = 128, 16
    P = 3 * k
    inv = O.rope_inv_freq(k)
    pos = np.array([[2.0, 3.0, 5.0]])
    ang = O.rope_angles(pos, inv)
    assert ang.shape == (1, P)
    # axis-major: angle[axis*k + j] = pos[axis] * inv[j]
    assert ang[0, 0] == 2.0 and ang[0, k] == 3.0 and ang[0, 2 * k] == 5.0
    assert ang[0, k + 1] == pytest.approx(3.0 * 10000 ** (-1 / 16))
    for j in (0, 17, 40):
        e = np.zeros((1, 1, hd))
        e[0, 0, j] = 1.0
        y = O.qk_norm_rope(e, np.ones(hd), ang, 0.0)[0, 0]
        s = math.sqrt(hd)                               # rms of a unit basis vector is 1/sqrt(hd)
        a = ang[0, j]
        assert y[j] == pytest.approx(s * math.cos(a), abs=1e-12)
        assert y[j + P] == pytest.approx(s * math.sin(a), abs=1e-12)
        others = np.delete(y, [j, j + P])
        assert np.abs(others).max() == 0.0
        # the partner rotates the other way: (0, 1) -> (-sin, cos)
        e2 = np.zeros((1, 1, hd))
        e2[0, 0, j + P] = 1.0
        y2 = O.qk_norm_rope(e2, np.ones(hd), ang, 0.0)[0, 0]
        assert y2[j] == pytest.approx(-s * math.sin(a), abs=1e-12)
        assert y2[j + P] == pytest.approx(s * math.cos(a), abs=1e-12)


def test_rope_norm_identity_relative_position_and_untouched_tail():
    rng = np.random.default_rng(5)
    hd, k = 128, 16
    inv = O.rope_inv_freq(k)
    v = rng.standard_normal((6, 3, hd))
    g = np.ones(hd)
    pos = rng.uniform(0, 300, (6, 3))
    y0 = O.qk_norm_rope(v, g, O.rope_angles(np.zeros((6, 3)), inv), 1e-5)
    np.testing.assert_allclose(y0, O.rms_norm(v, g, 1e-5), atol=1e-13)   # pos 0: identity
    y = O.qk_norm_rope(v, g, O.rope_angles(pos, inv), 1e-5)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(y0, axis=-1), rtol=1e-12)
    np.testing.assert_array_equal(y[..., 96:], y0[..., 96:])              # dims >= 96 untouched

    # q.k depends only on the position difference: shift every axis by
    # delta.  The rotation is checked with exact (unrounded) angles, which
    # are linear in the position; rope_angles' f32 rounding is pinned on its
    # own below.
    def exact_angles(p):
        return (p[:, :, None] * inv[None, None, :]).reshape(p.shape[0], -1)

    ye = O.qk_norm_rope(v, g, exact_angles(pos), 1e-5)
    for delta in ([7.0, 0, 0], [0, -3.5, 0], [0, 0, 11.25]):
        ys = O.qk_norm_rope(v, g, exact_angles(pos + np.array(delta)), 1e-5)
        dots = np.einsum("ahd,bhd->abh", ye, ye)
        dots_s = np.einsum("ahd,bhd->abh", ys, ys)
        np.testing.assert_allclose(dots, dots_s, atol=1e-9)


def test_rope_angles_are_f32_roundings_of_the_product():
    # The page stores the frequencies as an f32 tensor and every angle as
    # f32: each angle must be an f32 value, within half an f32 ulp of the
    # exact product of the position and the f32 frequency, and the angles
    # of integer positions on the first frequency (1.0) stay exact.
    rng = np.random.default_rng(9)
    k = 16
    inv = O.rope_inv_freq(k)
    pos = np.concatenate([rng.uniform(0, 700, (50, 3)), np.arange(12.0).reshape(4, 3)])
    ang = O.rope_angles(pos, inv)
    assert np.array_equal(ang.astype(np.float32).astype(np.float64), ang)
    inv32 = np.array([float(np.float32(f)) for f in inv])
    for i in range(pos.shape[0]):
        for a in range(3):
            for j in range(k):
                exact = pos[i, a] * inv32[j]
                got = ang[i, a * k + j]
                ulp = float(np.spacing(np.float32(abs(exact)))) if exact != 0 else 0.0
                assert abs(got - exact) <= 0.5 * ulp
    np.testing.assert_array_equal(ang[-4:, 0::k], pos[-4:])
    # the f32 frequencies differ from the fp64 formula by at most half an f32 ulp
    assert np.all(np.abs(inv32 - inv) <= 0.5 * np.spacing(inv.astype(np.float32)).astype(np.float64))


# --------------------------------------------------------------- attention

def _attention_loops(q, k, v, scale):
    n, nh, hd = q.shape
    out = np.zeros_like(v)
    for h in range(nh):
        for i in range(n):
            s = [scale * sum(q[i, h, d] * k[j, h, d] for d in range(hd)) for j in range(n)]
            m = max(s)
            e = [math.exp(x - m) for x in s]
            den = sum(e)
            for d in range(hd):
                out[i, h, d] = sum(e[j] * v[j, h, d] for j in range(n)) / den
    return out


def test_attention_brute_force_and_special_cases():
    rng = np.random.default_rng(6)
    q, k, v = (rng.standard_normal((5, 2, 4)) for _ in range(3))
    np.testing.assert_allclose(O.attention(q, k, v, 0.5), _attention_loops(q, k, v, 0.5), atol=1e-13)
    # one token: O = v
    np.testing.assert_allclose(O.attention(q[:1], k[:1], v[:1], 1.0), v[:1], atol=1e-15)
    # constant values: O = v
    vc = np.broadcast_to(rng.standard_normal((1, 2, 4)), (5, 2, 4))
    np.testing.assert_allclose(O.attention(q, k, vc, 1.0), vc, atol=1e-13)
    # softmax rows sum to one and permutation equivariance
    p = O.softmax_rows(rng.standard_normal((4, 9)) * 30)
    np.testing.assert_allclose(p.sum(-1), 1.0, atol=1e-14)
    perm = rng.permutation(5)
    np.testing.assert_allclose(O.attention(q[perm], k[perm], v[perm], 0.3),
                               O.attention(q, k, v, 0.3)[perm], atol=1e-13)
    # sampled query rows equal the full computation's rows
    np.testing.assert_allclose(O.attention(q, k, v, 0.3, q_rows=[4, 1]),
                               O.attention(q, k, v, 0.3)[[4, 1]], atol=1e-15)


# ------------------------------------------------------------------- block

def _tiny_block_inputs(seed=7, n=6, H=8, nh=2, hd=8, F=8):
    rng = np.random.default_rng(seed)
    I = nh * hd
    p = dict(norm1=1 + 0.1 * rng.standard_normal(H), norm2=1 + 0.1 * rng.standard_normal(H),
             wqkv=0.3 * rng.standard_normal((3 * I, H)), wout=0.3 * rng.standard_normal((H, I)),
             q_norm=1 + 0.1 * rng.standard_normal(hd), k_norm=1 + 0.1 * rng.standard_normal(hd),
             wfc1=0.3 * rng.standard_normal((2 * F, H)), wfc2=0.3 * rng.standard_normal((H, F)))
    dims = dict(hidden=H, heads=nh, head_dim=hd, ffn=F, eps=1e-5, qk_eps=1e-5,
                rope_k=hd // 8, rope_theta=10000.0)
    x = rng.standard_normal((n, H))
    mods = 0.3 * rng.standard_normal((6, 6 * H))
    rows = np.array([1, 1, 5, 5, 0, 0])[:n]
    pos = rng.uniform(0, 20, (n, 3))
    return p, dims, x, mods, rows, pos


def _block_loops(p, dims, x, mods, rows, pos):
    """The block written out element by element from mmh3.rs block_forward /
    ffn_tail / norm_rope_w, without matrix routines."""
    H, nh, hd, F = dims["hidden"], dims["heads"], dims["head_dim"], dims["ffn"]
    I = nh * hd
    n = x.shape[0]
    kf = dims["rope_k"]
    P = 3 * kf
    # the page's rope_angles: f32 frequencies, f64 product, f32 angle
    inv = [float(np.float32(dims["rope_theta"] ** (-i / kf))) for i in range(kf)]

    def rms(vec, g, eps):
        ss = sum(t * t for t in vec) / len(vec)
        r = 1 / math.sqrt(ss + eps)
        return [vec[i] * r * g[i] for i in range(len(vec))]

    def md(r, e):
        return [mods[rows[r]][e * H + j] for j in range(H)]

    def matvec(w, vec):
        return [sum(w[o][i] * vec[i] for i in range(len(vec))) for o in range(len(w))]

    xn = []
    for r in range(n):
        t = rms(list(x[r]), p["norm1"], dims["eps"])
        sh, sc = md(r, 0), md(r, 1)
        xn.append([t[j] * (1 + sc[j]) + sh[j] for j in range(H)])
    qkv = [matvec(p["wqkv"], xn[r]) for r in range(n)]
    Q = np.zeros((n, nh, hd)); K = np.zeros((n, nh, hd)); V = np.zeros((n, nh, hd))
    for r in range(n):
        ang = [float(np.float32(pos[r][a] * inv[j])) for a in range(3) for j in range(kf)]
        for h in range(nh):
            for which, dst, w in ((0, Q, p["q_norm"]), (1, K, p["k_norm"])):
                seg = qkv[r][which * I + h * hd: which * I + (h + 1) * hd]
                y = rms(seg, w, dims["qk_eps"])
                for j in range(P):
                    c, s = math.cos(ang[j]), math.sin(ang[j])
                    lo, hi = y[j], y[j + P]
                    y[j], y[j + P] = lo * c - hi * s, lo * s + hi * c
                dst[r, h] = y
            V[r, h] = qkv[r][2 * I + h * hd: 2 * I + (h + 1) * hd]
    att = _attention_loops(Q, K, V, 1 / math.sqrt(hd)).reshape(n, I)
    out = np.zeros((n, H))
    for r in range(n):
        proj = matvec(p["wout"], list(att[r]))
        g2 = md(r, 2)
        xm = [x[r][j] + g2[j] * proj[j] for j in range(H)]
        t = rms(xm, p["norm2"], dims["eps"])
        sh, sc = md(r, 3), md(r, 4)
        x2 = [t[j] * (1 + sc[j]) + sh[j] for j in range(H)]
        gu = matvec(p["wfc1"], x2)
        a = [gu[f] / (1 + math.exp(-gu[f])) * gu[F + f] for f in range(F)]
        d = matvec(p["wfc2"], a)
        g5 = md(r, 5)
        out[r] = [xm[j] + g5[j] * d[j] for j in range(H)]
    return out


def test_block_matches_elementwise_loops():
    p, dims, x, mods, rows, pos = _tiny_block_inputs()
    ref = _block_loops(p, dims, x, mods, rows, pos)
    np.testing.assert_allclose(O.block_forward(p, x, mods, rows, pos, dims), ref, atol=1e-12)


def test_block_zero_gates_is_identity_and_sampled_rows_agree():
    p, dims, x, mods, rows, pos = _tiny_block_inputs(seed=8)
    H = dims["hidden"]
    m0 = mods.copy()
    m0[:, 2 * H:3 * H] = 0
    m0[:, 5 * H:6 * H] = 0
    np.testing.assert_array_equal(O.block_forward(p, x, m0, rows, pos, dims), x)
    full = O.block_forward(p, x, mods, rows, pos, dims)
    np.testing.assert_allclose(O.block_forward(p, x, mods, rows, pos, dims, sample_rows=[5, 0, 3]),
                               full[[5, 0, 3]], atol=1e-13)


def test_block_in_chunks_with_kv_cache_equals_the_whole_block():
    # the block computed in chunks of query rows, k and v computed once by
    # the first chunk and read back by the others, gives the whole block
    p, dims, x, mods, rows, pos = _tiny_block_inputs()
    full = O.block_forward(p, x, mods, rows, pos, dims)
    cache = {}
    n = x.shape[0]
    parts = [O.block_forward(p, x, mods, rows, pos, dims, sample_rows=np.arange(a, min(a + 5, n)),
                             kv_cache=cache) for a in range(0, n, 5)]
    assert set(cache) == {"k", "v"} and cache["k"].shape[0] == n
    # equal up to the summation order the matrix product picks for a row count
    np.testing.assert_allclose(np.concatenate(parts), full, rtol=0, atol=1e-12)


def test_block_zero_shift_scale_reduces_to_plain_rmsnorm():
    p, dims, x, mods, rows, pos = _tiny_block_inputs(seed=9)
    H = dims["hidden"]
    keep = {}
    m = mods.copy()
    m[:, 0:2 * H] = 0
    O.block_forward(p, x, m, rows, pos, dims, keep=keep)
    np.testing.assert_allclose(keep["xn1"], O.rms_norm(x, p["norm1"], 1e-5), atol=1e-15)


def test_unmodulated_block_uses_plain_residual():
    p, dims, x, mods, rows, pos = _tiny_block_inputs(seed=10)
    H = dims["hidden"]
    ones = np.zeros_like(mods)
    ones[:, 2 * H:3 * H] = 1
    ones[:, 5 * H:6 * H] = 1
    np.testing.assert_allclose(O.block_forward(p, x, None, rows, pos, dims),
                               O.block_forward(p, x, ones, rows, pos, dims), atol=1e-13)


def test_heads_sign_and_modulation():
    rng = np.random.default_rng(11)
    x = rng.standard_normal((4, 6))
    g = np.ones(6)
    w = np.eye(6)[:3]
    b = np.array([1.0, 2.0, 3.0])
    fm = np.zeros(12)
    y = O.heads_forward(x, g, fm, w, b, 0.0)
    np.testing.assert_allclose(y, -(O.rms_norm(x, g, 0.0)[:, :3] + b), atol=1e-14)
    fm[:6] = 0.5          # shift
    fm[6:] = 1.0          # scale: x*2 + 0.5
    y = O.heads_forward(x, g, fm, w, b, 0.0)
    np.testing.assert_allclose(y, -(2 * O.rms_norm(x, g, 0.0)[:, :3] + 0.5 + b), atol=1e-14)


# ------------------------------------------------------------------ SigLIP

def test_vit_layer_against_loops_and_scale_fold():
    rng = np.random.default_rng(12)
    B, S, H, nh, hd, M = 2, 3, 4, 2, 2, 6
    p = dict(ln1_g=1 + 0.1 * rng.standard_normal(H), ln1_b=0.1 * rng.standard_normal(H),
             wo=0.5 * rng.standard_normal((H, H)), bo=0.1 * rng.standard_normal(H),
             ln2_g=1 + 0.1 * rng.standard_normal(H), ln2_b=0.1 * rng.standard_normal(H),
             w1=0.5 * rng.standard_normal((M, H)), b1=0.1 * rng.standard_normal(M),
             w2=0.5 * rng.standard_normal((H, M)), b2=0.1 * rng.standard_normal(H))
    wq, wk, wv = (0.5 * rng.standard_normal((H, H)) for _ in range(3))
    bq, bk, bv = (0.1 * rng.standard_normal(H) for _ in range(3))
    fq, fb = O.vit_fold_scale(wq, bq, hd)
    p["wqkv"] = np.concatenate([fq, wk, wv])
    p["bqkv"] = np.concatenate([fb, bk, bv])
    dims = dict(hidden=H, heads=nh, head_dim=hd, mlp=M, ln_eps=1e-6)
    x = rng.standard_normal((B * S, H))
    got = O.vit_layer_forward(p, x, B, S, dims)
    # loops, with the scale applied to the product instead of folded
    ref = np.zeros_like(x)
    for bi in range(B):
        xi = x[bi * S:(bi + 1) * S]

        def ln(v, g, bb):
            mu = sum(v) / H
            var = sum((t - mu) ** 2 for t in v) / H
            return [(v[j] - mu) / math.sqrt(var + 1e-6) * g[j] + bb[j] for j in range(H)]
        hn = [ln(list(r), p["ln1_g"], p["ln1_b"]) for r in xi]
        q = np.array([[sum(wq[o][i] * r[i] for i in range(H)) + bq[o] for o in range(H)] for r in hn])
        kk = np.array([[sum(wk[o][i] * r[i] for i in range(H)) + bk[o] for o in range(H)] for r in hn])
        vv = np.array([[sum(wv[o][i] * r[i] for i in range(H)) + bv[o] for o in range(H)] for r in hn])
        o = _attention_loops(q.reshape(S, nh, hd), kk.reshape(S, nh, hd), vv.reshape(S, nh, hd),
                             1 / math.sqrt(hd)).reshape(S, H)
        for r in range(S):
            y = [xi[r][j] + sum(p["wo"][j][i] * o[r][i] for i in range(H)) + p["bo"][j] for j in range(H)]
            h2 = ln(y, p["ln2_g"], p["ln2_b"])
            a = []
            for m in range(M):
                z = sum(p["w1"][m][i] * h2[i] for i in range(H)) + p["b1"][m]
                a.append(0.5 * z * (1 + math.tanh(math.sqrt(2 / math.pi) * (z + 0.044715 * z ** 3))))
            ref[bi * S + r] = [y[j] + sum(p["w2"][j][m] * a[m] for m in range(M)) + p["b2"][j]
                               for j in range(H)]
    np.testing.assert_allclose(got, ref, atol=1e-12)
    # images are independent: computing one image alone gives its rows
    np.testing.assert_allclose(O.vit_layer_forward(p, x, B, S, dims, images=[1]), got[S:], atol=1e-15)


# --------------------------------------------------------------- generator

def test_splitmix64_published_values_and_tensor_form():
    # SplitMix64 seeded with 0: the first outputs of Vigna's reference code
    assert synth.splitmix64_scalar(0, 3) == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4,
                                             0x06C45D188009454F]
    for seed in (0, 1, 123456789, (1 << 64) - 5):
        ref = synth.splitmix64_scalar(seed, 40)
        t = synth.splitmix64(seed, 40)
        assert [int(v) & ((1 << 64) - 1) for v in t] == ref
        t2 = synth.splitmix64(seed, 10, start=30)
        assert [int(v) & ((1 << 64) - 1) for v in t2] == ref[30:]


def test_gauss_pairs_and_moments():
    u = [(z >> 11) / float(1 << 53) for z in synth.splitmix64_scalar(42, 4)]
    r = math.sqrt(-2 * math.log(max(u[0], 1e-300)))
    g = synth.gauss(3, 42)
    assert g[0].item() == pytest.approx(r * math.cos(2 * math.pi * u[1]), rel=1e-15)
    assert g[1].item() == pytest.approx(r * math.sin(2 * math.pi * u[1]), rel=1e-15)
    big = synth.gauss(1 << 20, 7)
    assert abs(big.mean().item()) < 5e-3 and abs(big.std().item() - 1) < 5e-3
    # chunking does not change the stream
    assert torch.equal(synth.gauss(10, 9), synth.gauss(11, 9)[:10])
    random.seed(0)


# ------------------------------------------------------- refiner and embed

def test_patchify_and_audio_pack_round_trip_page_tests():
    # mmh3.rs tests patchify_round_trips / audio_pack_round_trips
    c, t, h, w = 3, 2, 4, 6
    x = np.arange(c * t * h * w, dtype=np.float64).reshape(c, t, h, w)
    rows = O.patchify_video(x)
    assert rows.shape == (t * (h // 2) * (w // 2), c * 4)
    np.testing.assert_array_equal(O.unpatchify_video(rows, c, t, h, w), x)
    ca, ta = 5, 7
    xa = np.arange(ca * 2 * ta, dtype=np.float64).reshape(ca, 2, ta)
    np.testing.assert_array_equal(O.unpack_audio(O.pack_audio(xa), ca, ta), xa)


def test_patchify_element_order_by_hand():
    # row (t, hi, wi), column (c, p, q) holds x[c, t, 2 hi + p, 2 wi + q]
    c, t, h, w = 2, 3, 4, 6
    x = np.random.default_rng(13).standard_normal((c, t, h, w))
    rows = O.patchify_video(x)
    for (ti, hi, wi) in ((0, 0, 0), (2, 1, 2), (1, 1, 0)):
        r = (ti * (h // 2) + hi) * (w // 2) + wi
        for ci in range(c):
            for p in range(2):
                for q in range(2):
                    assert rows[r, ci * 4 + p * 2 + q] == x[ci, ti, 2 * hi + p, 2 * wi + q]
    xa = np.random.default_rng(14).standard_normal((4, 2, 5))
    pa = O.pack_audio(xa)
    assert pa[0, 3] == xa[3, 0, 0] and pa[5 + 2, 1] == xa[1, 1, 2]   # channel-major rows


def test_refine_text_without_blocks_is_projection_then_rmsnorm():
    rng = np.random.default_rng(15)
    s = rng.standard_normal((5, 6))
    w = rng.standard_normal((4, 6))
    b = rng.standard_normal(4)
    g = 1 + 0.1 * rng.standard_normal(4)
    out = O.refine_text(s, w, b, [], g, dict(hidden=4), 1e-5)
    h = np.array([[sum(s[i, k] * w[o, k] for k in range(6)) + b[o] for o in range(4)] for i in range(5)])
    ref = h / np.sqrt((h * h).mean(-1, keepdims=True) + 1e-5) * g
    np.testing.assert_allclose(out, ref, atol=1e-12)


def test_embed_places_each_stream_in_its_segment():
    L = O.layout_t2va(3, 2, 4, 4, 2)                 # text 3, audio 2x2, video 2x2x2
    n = L["seq_len"]
    rng = np.random.default_rng(16)
    H = 5
    text = rng.standard_normal((3, H))
    video = rng.standard_normal((2, 2, 4, 4))        # C=2 -> 4C = 8
    audio = rng.standard_normal((3, 2, 2))           # C=3
    wv, bv = rng.standard_normal((H, 8)), rng.standard_normal(H)
    wa, ba = rng.standard_normal((H, 3)), rng.standard_normal(H)
    h = O.embed(L, text, video, audio, wv, bv, wa, ba)
    assert h.shape == (n, H)
    np.testing.assert_array_equal(h[:3], text)
    # first audio row = channel 0, frame 0 of every latent channel, projected
    np.testing.assert_allclose(h[3], wa @ audio[:, 0, 0] + ba, atol=1e-12)
    # first video row = the 2x2 patch at the top-left of frame 0
    np.testing.assert_allclose(h[7], wv @ video[:, 0, 0:2, 0:2].reshape(-1) + bv, atol=1e-12)


def test_embed_condition_frames_use_the_patch_projection():
    # a segment table [text | cond frame | target video]: the condition frame
    # is one latent frame through the video patch projection
    rng = np.random.default_rng(17)
    H, C = 4, 1
    L = {"seq_len": 2 + 4 + 8,
         "segments": [(0, 2, O.TAG_TEXT, 0), (2, 6, O.TAG_VIDEO, 0), (6, 14, O.TAG_VIDEO, 0)]}
    text = rng.standard_normal((2, H))
    video = rng.standard_normal((C, 2, 4, 4))
    cond = rng.standard_normal((C, 1, 4, 4))
    wv, bv = rng.standard_normal((H, 4 * C)), rng.standard_normal(H)
    h = O.embed(L, text, video, np.zeros((1, 2, 0)), wv, bv, np.zeros((H, 1)), np.zeros(H), cond=[cond])
    # condition row 3 = patch (h=0, w=1) of the condition frame
    np.testing.assert_allclose(h[3], wv @ cond[0, 0, 0:2, 2:4].reshape(-1) + bv, atol=1e-12)
    # target row 6 + 4 = frame 1, patch (0, 0)
    np.testing.assert_allclose(h[10], wv @ video[0, 1, 0:2, 0:2].reshape(-1) + bv, atol=1e-12)
    np.testing.assert_array_equal(h[:2], text)


def test_denoise_forward_identity_weights_return_the_negated_latents():
    # H = 4 C_v = C_a; identity patch projections and head linears, no bias,
    # zero final modulation, unit final gain, no blocks: every packed row is
    # RMS-normalised and mapped back, so latents of +-1 (RMS exactly 1) come
    # back negated through patchify -> heads -> unpatchify (and the audio
    # pack / unpack) -- any transposition in the chain breaks this.
    H, Cv, Ca = 8, 2, 8
    L = O.layout_t2va(3, 2, 4, 6, 5)
    rng = np.random.default_rng(21)
    video = rng.choice([-1.0, 1.0], size=(Cv, 2, 4, 6))
    audio = rng.choice([-1.0, 1.0], size=(Ca, 2, 5))
    text = rng.standard_normal((3, H))
    eye = np.eye(H)
    heads = {"final_norm": np.ones(H), "adaln_w": np.zeros((2 * 2 * H, 24)),
             "adaln_b": np.zeros(2 * 2 * H), "adaln_table": rng.standard_normal((1025, 24)),
             "w_video": eye, "b_video": np.zeros(H), "w_audio": eye, "b_audio": np.zeros(H)}
    dims = {"hidden": H, "eps": 1e-300}
    v, a = O.denoise_forward(L, text, video, audio, (eye, np.zeros(H), eye, np.zeros(H)), [],
                             heads, 0.5, 0.2, dims)
    np.testing.assert_allclose(v, -video, rtol=0, atol=1e-14)
    np.testing.assert_allclose(a, -audio, rtol=0, atol=1e-14)


def test_denoise_forward_each_stream_reads_its_own_clocks_final_row():
    # Same identity chain, now with a final-layer bias whose scale chunk is
    # 1 in slot 0 and 3 in slot 1 (zero basis).  sigma_v 0.5 and sigma_a 0.2
    # give ts = [0.5, 0.8]: the video clock owns slot 0 (x * 2) and the audio
    # clock slot 1 (x * 4).  Swapping the streams' final rows, or the slot
    # order inside final_mods, swaps the factors.
    H, Cv, Ca = 8, 2, 8
    L = O.layout_t2va(3, 2, 4, 6, 5)
    rng = np.random.default_rng(22)
    video = rng.choice([-1.0, 1.0], size=(Cv, 2, 4, 6))
    audio = rng.choice([-1.0, 1.0], size=(Ca, 2, 5))
    text = rng.standard_normal((3, H))
    eye = np.eye(H)
    b = np.zeros(2 * 2 * H)
    b[H:2 * H] = 1.0            # slot 0 scale
    b[3 * H:4 * H] = 3.0        # slot 1 scale
    heads = {"final_norm": np.ones(H), "adaln_w": np.zeros((2 * 2 * H, 24)),
             "adaln_b": b, "adaln_table": rng.standard_normal((1025, 24)),
             "w_video": eye, "b_video": np.zeros(H), "w_audio": eye, "b_audio": np.zeros(H)}
    dims = {"hidden": H, "eps": 1e-300}
    ts, slot = O.plan_timesteps(0.5, 0.2, L["segments"])
    assert ts == [0.5, 0.8] and slot == {O.CLOCK_VIDEO: 0, O.CLOCK_AUDIO: 1}
    v, a = O.denoise_forward(L, text, video, audio, (eye, np.zeros(H), eye, np.zeros(H)), [],
                             heads, 0.5, 0.2, dims)
    np.testing.assert_allclose(v, -2.0 * video, rtol=0, atol=1e-14)
    np.testing.assert_allclose(a, -4.0 * audio, rtol=0, atol=1e-14)


# ------------------------------------------------- keyframe / reference layouts

def test_keyframes_sit_between_the_text_and_the_audio_page_test():
    # "cortiq_engine/mmh3.rs" test keyframes_sit_between_the_text_and_the_audio:
    # t2va(8, 3, 8, 12, 5) against fl2va with the first and last frame of a
    # 39-frame clip
    tl, lt, lh, lw, at = 8, 3, 8, 12, 5
    base = O.layout_t2va(tl, lt, lh, lw, at)
    L = O.layout_fl2va(tl, lt, lh, lw, at, [(0, 39), (38, 39)])
    cond = [s for s, k in zip(L["segments"], L["kinds"]) if k == "Cond"]
    assert sum(b - a for a, b, _, _ in cond) == 2 * L["frame_rows"] == 48
    assert L["seq_len"] == base["seq_len"] + 2 * L["frame_rows"] == 138
    assert L["kinds"] == ["Text", "Cond", "Cond", "Audio", "Video"]
    seg = {k: s for s, k in zip(L["segments"], L["kinds"])}
    bseg = dict(zip(base["kinds"], base["segments"]))
    # a keyframe never advances the cursor
    assert L["pos"][seg["Audio"][0], 0] == base["pos"][bseg["Audio"][0], 0]
    assert L["pos"][seg["Video"][0], 0] == base["pos"][bseg["Video"][0], 0]
    # first frame at the text's end, the last a whole clip further, minus one span
    assert L["pos"][cond[0][0], 0] == tl
    spans = sum(O.FRAME_RESCALE * O.FRAME_PER_TOKEN[k % 5] for k in range(lt))
    assert abs(L["pos"][cond[1][0], 0] - (tl + spans - O.FRAME_RESCALE)) < 1e-12
    assert abs(L["pos"][cond[1][0], 0] - (8 + 15 - 5 / 3)) < 1e-12           # spans = 5/3 (1+4+4)
    # both keyframes share the target grid
    np.testing.assert_array_equal(L["pos"][cond[0][0]:cond[0][1], 1:], L["pos"][seg["Video"][0]:seg["Video"][0] + 24, 1:])
    # keyframe rows: tag video on the visual condition clock
    assert all(s[2] == O.TAG_VIDEO and s[3] == O.CLOCK_COND for s in cond)
    with pytest.raises(ValueError):
        O.layout_fl2va(tl, lt, lh, lw, at, [(5, 39)])


def test_reference_blocks_advance_the_cursor_by_hand():
    # a still: its own grid at the cursor, cursor + 1
    L = O.layout_ref2va(4, 2, 4, 4, 3, [("image", 4, 6)])
    assert L["kinds"] == ["Text", "RefImg", "Audio", "Video"]
    img = L["segments"][1]
    assert img[1] - img[0] == 2 * 3 and (img[2], img[3]) == (O.TAG_VIDEO, O.CLOCK_COND)
    assert (L["pos"][img[0]:img[1], 0] == 4.0).all()
    a = math.sqrt(24)
    assert L["pos"][img[0] + 1, 2] == O.axis_from_sqrt_area(6, 2, a)[1]
    assert L["pos"][L["segments"][2][0], 0] == 5.0 and L["pos"][L["segments"][3][0], 0] == 5.0
    # standalone audio: t stereo frames from the cursor (target grid's w extremes), cursor + t
    L = O.layout_ref2va(4, 2, 4, 4, 3, [("audio", 3)])
    ra = L["segments"][1]
    assert L["kinds"][1] == "RefAudio" and (ra[2], ra[3]) == (O.TAG_AUDIO, O.CLOCK_COND_AUDIO)
    np.testing.assert_array_equal(L["pos"][ra[0]:ra[1], 0], [4, 5, 6, 4, 5, 6])
    w_t = O.axis_from_sqrt_area(4, 2, 4.0)
    assert L["pos"][ra[0], 2] == w_t[0] and L["pos"][ra[1] - 1, 2] == w_t[-1]
    assert L["pos"][L["segments"][2][0], 0] == 7.0
    # a clip: soundtrack first (its own w extremes), frames stepping by the
    # spans, cursor + max(audio frames, spans)
    L = O.layout_ref2va(4, 2, 4, 4, 3, [("video", 2, 4, 8, 5)])
    assert L["kinds"] == ["Text", "RefAudio", "RefImg", "Audio", "Video"]
    ra, rv = L["segments"][1], L["segments"][2]
    w_r = O.axis_from_sqrt_area(8, 2, math.sqrt(32))
    assert L["pos"][ra[0], 2] == w_r[0] and L["pos"][ra[1] - 1, 2] == w_r[-1]
    assert L["pos"][rv[0], 0] == 4.0 and abs(L["pos"][rv[0] + 8, 0] - (4 + 5 / 3)) < 1e-12
    assert abs(L["pos"][L["segments"][3][0], 0] - (4 + 25 / 3)) < 1e-12   # max(5, 5/3 + 20/3)
    # a clip whose soundtrack is longer than its frames
    L = O.layout_ref2va(4, 2, 4, 4, 3, [("video", 1, 4, 4, 5)])
    assert L["pos"][L["segments"][3][0], 0] == 9.0                          # max(5, 5/3)


def test_condition_rows_hand_enumerated():
    # fl2va at sigma_v 0.3: t_v 0.7, t_a 28/31, t_cond max(0.7, 0.999)
    L = O.layout_fl2va(8, 3, 8, 12, 5, [(0, 39)])
    sa = O.time_shift_sigma(0.3, 12, 3)
    ts, slot = O.plan_timesteps(0.3, sa, L["segments"])
    np.testing.assert_allclose(ts, [0.7, 28 / 31, 0.999], rtol=0, atol=1e-15)
    rows = O.token_rows(L["segments"], slot, L["seq_len"])
    assert [int(rows[s[0]]) for s in L["segments"]] == [1, 6, 5, 0]
    # late in sampling t_v passes 0.999: the keyframes share the video slot
    sv = 1e-4
    sa = O.time_shift_sigma(sv, 12, 3)
    ts, slot = O.plan_timesteps(sv, sa, L["segments"])
    assert len(ts) == 2 and slot[O.CLOCK_COND] == slot[O.CLOCK_VIDEO] == 0
    rows = O.token_rows(L["segments"], slot, L["seq_len"])
    assert [int(rows[s[0]]) for s in L["segments"]] == [1, 0, 5, 0]
    # ref2va with a still and standalone audio: four clocks, four timesteps
    L = O.layout_ref2va(4, 2, 4, 4, 3, [("image", 4, 4), ("audio", 2)])
    ts, slot = O.plan_timesteps(0.3, O.time_shift_sigma(0.3, 12, 3), L["segments"])
    assert len(ts) == 4 and ts[-2:] == [0.999, 1.0]
    rows = O.token_rows(L["segments"], slot, L["seq_len"])
    assert [int(rows[s[0]]) for s in L["segments"]] == [1, 6, 11, 5, 0]


def test_text_tags_split_the_prompt_into_runs():
    L = O.layout_fl2va(8, 1, 4, 4, 2, [], text_tags=[1, 1, 0, 0, 1, 1, 1, 1])
    assert L["segments"][:3] == [(0, 2, 1, 0), (2, 4, 0, 0), (4, 8, 1, 0)]
    ts, slot = O.plan_timesteps(0.5, 0.2, L["segments"])
    rows = O.token_rows(L["segments"], slot, L["seq_len"])
    assert list(rows[:8]) == [1, 1, 0, 0, 1, 1, 1, 1]
