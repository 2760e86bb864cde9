"""Full-size stack and image workloads on the GPU.

The oracle cannot run 50 full-size blocks in fp64, so the stack is checked
through properties that hold at any size plus oracle parity on sampled rows:
  * with every block's gates zero, the 50-block stack leaves x exactly
    unchanged, and both output heads then match the oracle's heads on the
    (unchanged) input rows;
  * the stack call equals 50 separate block calls bit for bit;
  * one image-mode block at full size (one clock, two tags) matches the
    oracle on sampled rows, and the image head (target rows) does too.
"""

import pytest

from gpu_common import (BF16_STORE_REL, O, api, assert_close, configs, f64, np, oracle_block,
                        run_block, sigma_pair, t2va, torch)

pytestmark = pytest.mark.gpu


def _zero_gates(w, H):
    """Zero the gate chunks (2: gate_msa, 5: gate_mlp) of every adaLN row."""
    for e in (2, 5):
        for r in range(6):
            lo = r * 6 * H + e * H
            w["adaln_w"][lo:lo + H] = 0
            w["adaln_b"][lo:lo + H] = 0


def _stack_inputs(c, dev="cuda"):
    segs, pos = api.layout_t2va(c.text_len, c.latent_t, c.lat_h, c.lat_w, c.audio_t)
    dims = api.make_dims(c.hidden, c.heads, c.head_dim, c.ffn)
    return segs, pos, dims


def test_stack_full_size_zero_gates_identity_and_heads(cuda_ok):
    c = configs.STACK
    segs, pos, dims = _stack_inputs(c)
    n = pos.shape[0]
    assert n == 26496
    blocks = []
    for b in range(c.n_blocks):
        w = configs.block_weights(c, b, device="cuda")
        _zero_gates(w, c.hidden)
        blocks.append(api.BlockParams.from_host(dims, w, device="cuda"))
    hw = configs.head_weights(c)
    heads = api.HeadParams.from_host(hw)
    x = configs.hidden_states(c)
    xd = x.cuda()
    pd = torch.as_tensor(pos.astype(np.float32)).cuda()
    sv, sa = sigma_pair(c.sigma_v)
    vs = [s for s in segs if s[2] == 0][-1]
    as_ = [s for s in segs if s[2] == 2][-1]
    ov = torch.full((vs[1] - vs[0], 128), float("nan"), device="cuda")
    oa = torch.full((as_[1] - as_[0], 128), float("nan"), device="cuda")
    ws = torch.empty(api.workspace_size(dims, n), dtype=torch.uint8, device="cuda")
    api.stack_forward(dims, blocks, heads, xd, segs, pd, sv, sa, ov, oa, ws)
    api.device_status()
    assert torch.equal(xd.cpu(), x), "zero gates must leave the residual stream unchanged"
    # heads on sampled rows of each stream, from the oracle on the input rows
    ts, slot = O.plan_timesteps(sv, sa, segs)
    fm = O.final_mods(f64(hw["adaln_w"]), f64(hw["adaln_b"]), f64(hw["adaln_table"]), ts, c.hidden)
    for (seg, key, out) in ((vs, "video", ov), (as_, "audio", oa)):
        rows = np.linspace(seg[0], seg[1] - 1, 9).astype(int)
        ref = O.heads_forward(f64(x[rows]), f64(hw["final_norm"]), fm[slot[seg[3]]],
                              f64(hw[f"w_{key}"]), f64(hw[f"b_{key}"]), c.eps)
        assert_close(out[rows - seg[0]], ref, what=f"{key} head rows", rel=BF16_STORE_REL)


def test_stack_full_size_equals_separate_block_calls(cuda_ok):
    c = configs.STACK
    segs, pos, dims = _stack_inputs(c)
    n = pos.shape[0]
    blocks = [api.BlockParams.from_host(dims, configs.block_weights(c, b, device="cuda"), device="cuda")
              for b in range(c.n_blocks)]
    x = configs.hidden_states(c, device="cuda")
    pd = torch.as_tensor(pos.astype(np.float32)).cuda()
    sv, sa = sigma_pair(c.sigma_v)
    ws = torch.empty(api.workspace_size(dims, n), dtype=torch.uint8, device="cuda")
    x1 = x.clone()
    api.stack_forward(dims, blocks, None, x1, segs, pd, sv, sa, None, None, ws)
    x2 = x.clone()
    for b in blocks:
        api.block_forward(dims, b, x2, segs, pd, sv, sa, ws)
    api.device_status()
    assert torch.equal(x1, x2)
    assert torch.isfinite(x1).all()
    # fifty blocks move the residual stream but keep it bounded
    d = (x1 - x).float()
    assert 0 < d.abs().max().item() < 1e3


def test_image_block_full_size_sampled_rows_and_head(cuda_ok):
    c = configs.IMAGE
    L = O.layout_image(c.text_len, c.ref_lat_h, c.ref_lat_w, c.lat_h, c.lat_w)
    segs, pos, n = L["segments"], L["pos"], L["seq_len"]
    assert n == 8448
    w = configs.block_weights(c, 0)
    x = configs.hidden_states(c)
    sv, sa = sigma_pair(c.sigma_v)
    dims_c = api.make_dims(c.hidden, c.heads, c.head_dim, c.ffn)
    xg, reg = run_block(dims_c, w, x, segs, pos, sv, sa)
    sample = [0, 255, 256, 2000, 4351, 4352, 6000, 8447]
    keep = {}
    ref, mods, rows = oracle_block(w, x, segs, pos, sv, sa, c.dims(), sample_rows=sample, keep=keep)
    assert sorted(set(rows.tolist())) == [0, 1]
    assert_close(xg[sample], ref, what="image block rows")
    assert_close(xg[sample].cpu().double() - x[sample].double(), ref - f64(x[sample]), what="image block delta")
    assert_close(reg["attn"][sample], keep["attn"], what="image attn rows", rel=BF16_STORE_REL)
