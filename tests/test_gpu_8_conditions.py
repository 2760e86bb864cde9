"""Keyframe (fl2va) and reference (ref2va) layouts on the GPU against the
oracle ("cortiq_engine/mmh3.rs", Layout::fl2va / ref2va / build_full and
the condition-row assignment of forward).

* The per-token adaLN rows, written by the device gather, equal the
  oracle's exactly (four clocks, text-tag runs).
* A keyframe block late in sampling, where the visual condition clock
  shares the video timestep (two timesteps), runs on the block's own adaLN
  curve and matches the oracle.
* A reference block with four distinct timesteps runs with the caller's
  modulation (mods_or_null) and matches the oracle on the same modulation;
  the stack, which evaluates the curve itself, refuses it.
"""

import pytest

from gpu_common import (O, api, assert_close, configs, f64, np, sigma_pair, small_block_weights,
                        small_dims, synth, torch)
from packed_multimodal_diffusion_b200 import _lib

pytestmark = pytest.mark.gpu

FL2VA = ((20, 3, 16, 20, 20), [(38, 39)], [1] * 5 + [0] * 10 + [1] * 5)
REF2VA = ((10, 3, 16, 20, 6), [("image", 8, 8), ("audio", 4), ("video", 3, 8, 12, 0), ("video", 1, 4, 4, 7)],
          [1, 1, 1, 0, 0, 0, 0, 1, 1, 1])


@pytest.mark.parametrize("sigma_v", [1e-4, 0.3, 1.0])
def test_condition_rows_exact_through_the_device_gather(cuda_ok, sigma_v):
    for L in (O.layout_fl2va(*FL2VA[0], FL2VA[1], text_tags=FL2VA[2]),
              O.layout_ref2va(*REF2VA[0], REF2VA[1], text_tags=REF2VA[2])):
        sv, sa = sigma_pair(sigma_v)
        ts, slot = O.plan_timesteps(sv, sa, L["segments"])
        ref = O.token_rows(L["segments"], slot, L["seq_len"])
        rows = torch.full((L["seq_len"],), -7, dtype=torch.int32, device="cuda")
        api.resolve_rows(L["segments"], L["seq_len"], sv, sa, rows)
        np.testing.assert_array_equal(rows.cpu().numpy(), ref)


def test_keyframe_block_two_timesteps_own_curve(cuda_ok):
    dims_o, dims_c = small_dims()
    L = O.layout_fl2va(*FL2VA[0], FL2VA[1], text_tags=FL2VA[2])
    segs, pos, n = L["segments"], L["pos"], L["seq_len"]
    sv, sa = sigma_pair(1e-4)
    ts, slot = O.plan_timesteps(sv, sa, segs)
    assert len(ts) == 2 and slot[O.CLOCK_COND] == slot[O.CLOCK_VIDEO]
    w = small_block_weights(101, 256, 2, 128, 512)
    x = configs.synth.normal((n, 256), 102, 1.0)
    rows = O.token_rows(segs, slot, n)
    mods = O.block_mods(f64(w["adaln_w"]), f64(w["adaln_b"]), f64(w["adaln_table"]), ts, 256)
    ref = O.block_forward({k: f64(v) for k, v in w.items()}, f64(x), mods, rows, pos, dims_o)
    params = api.BlockParams.from_host(dims_c, w)
    xd = x.cuda().clone()
    pd = torch.as_tensor(pos.astype(np.float32)).cuda()
    ws = torch.empty(api.workspace_size(dims_c, n), dtype=torch.uint8, device="cuda")
    api.block_forward(dims_c, params, xd, segs, pd, sv, sa, ws)
    assert api.status_sync() == 0
    assert_close(xd, ref, what="keyframe block x_out")
    assert_close(xd.cpu().double() - x.double(), ref - f64(x), what="keyframe block delta")


def test_reference_block_four_timesteps_with_caller_modulation(cuda_ok):
    dims_o, dims_c = small_dims()
    L = O.layout_ref2va(*REF2VA[0], REF2VA[1], text_tags=REF2VA[2])
    segs, pos, n = L["segments"], L["pos"], L["seq_len"]
    sv, sa = sigma_pair(0.3)
    ts, slot = O.plan_timesteps(sv, sa, segs)
    assert len(ts) == 4
    rows = O.token_rows(segs, slot, n)
    assert sorted(set(rows.tolist())) == [0, 1, 5, 6, 11]
    w = small_block_weights(103, 256, 2, 128, 512)
    x = configs.synth.normal((n, 256), 104, 1.0)
    # a modulation buffer [4 * 3, 6H]: seeded values of the adaLN output's scale
    mods = synth.normal((12, 6 * 256), 105, 0.1).double().numpy()
    ref = O.block_forward({k: f64(v) for k, v in w.items()}, f64(x), mods, rows, pos, dims_o)
    params = api.BlockParams.from_host(dims_c, {k: v for k, v in w.items() if not k.startswith("adaln")})
    xd = x.cuda().clone()
    pd = torch.as_tensor(pos.astype(np.float32)).cuda()
    ws = torch.empty(api.workspace_size(dims_c, n), dtype=torch.uint8, device="cuda")
    api.block_forward(dims_c, params, xd, segs, pd, sv, sa, ws, mods=torch.as_tensor(mods.astype(np.float32)).cuda())
    assert api.status_sync() == 0
    assert_close(xd, ref, what="reference block x_out")
    assert_close(xd.cpu().double() - x.double(), ref - f64(x), what="reference block delta")
    # the stack evaluates the two-slot curve itself: refused before any launch
    full = api.BlockParams.from_host(dims_c, w)
    with pytest.raises(_lib.Mmh3Error) as e:
        api.stack_forward(dims_c, [full], None, xd, segs, pd, sv, sa, None, None, ws)
    assert e.value.code == 5
