"""The stack against the oracle, with real gates ("cortiq_engine/mmh3.rs",
forward "blocks" and "heads").

* Teacher-forced at the full stack workload (26 496 tokens, 50 blocks) and
  the image workload (8 448 tokens, 50 blocks, one clock): the GPU stack runs
  to block i - 1, and the oracle computes block i on the GPU's own x_i for
  i in {0, 24, 49}, on sampled rows that span every segment and the ragged
  last tile (k and v for every token).  Block i's output and its delta meet
  the block bars.  After block 49 the output heads (video and audio; the
  image head on the target image) are compared on sampled rows.
* A whole 50-block chain at the tiny workload's shape (64 tokens), untruncated,
  in fp32 storage (tf32 GEMMs) and in bf16 storage, against the oracle's
  50-block chain.
"""

import pytest

from gpu_common import (BF16_STORE_REL, TF32_COS, TF32_MAXABS, O, api, assert_close,
                        configs, f64, np, sigma_pair, torch)

pytestmark = pytest.mark.gpu


def _sample_rows(segs, n):
    """Rows spanning every segment's first and last row, a few interior rows
    and the last (ragged) 128-row tile."""
    rows = {0, n - 1, n - 2, (n // 128) * 128, (n // 128) * 128 - 1}
    for (a, b, _t, _c) in segs:
        rows |= {a, b - 1, (a + b) // 2}
    rows |= {int(r) for r in np.linspace(0, n - 1, 7)}
    return sorted(r for r in rows if 0 <= r < n)


def _host_weights(c, i, bp: api.BlockParams) -> dict:
    """Block i's device weights as the oracle reads them; fc1 in its natural
    [gate | up] order is generated again on the device from the same stream
    (the block holds only the tiled copy)."""
    p = {k: f64(v) for k, v in bp.tensors.items() if k != "wfc1_tiled"}
    p["wfc1"] = f64(configs.block_weights(c, i, device="cuda", keys=("wfc1",))["wfc1"])
    return p


@pytest.mark.parametrize("workload", ["stack", "image"])
def test_stack_full_size_teacher_forced_blocks_and_heads(cuda_ok, workload):
    c = configs.CONFIGS[workload]
    if c.image_mode:
        # one clock, two tags; the head reads the target image's rows
        segs, pos = api.layout_image(c.text_len, c.ref_lat_h, c.ref_lat_w, c.lat_h, c.lat_w)
        hc = configs.DitConfig(c.name, c.cfg_seed, hidden=c.hidden, heads=c.heads, head_dim=c.head_dim,
                               ffn=c.ffn, text_len=c.text_len, heads_out=128)
    else:
        segs, pos = api.layout_t2va(c.text_len, c.latent_t, c.lat_h, c.lat_w, c.audio_t)
        hc = c
    n = pos.shape[0]
    assert n == {"stack": 26496, "image": 8448}[workload]
    dims = api.make_dims(c.hidden, c.heads, c.head_dim, c.ffn)
    blocks = [api.BlockParams.from_host(dims, configs.block_weights(c, b, device="cuda"), device="cuda")
              for b in range(c.n_blocks)]
    hw = configs.head_weights(hc, device="cuda")
    heads = api.HeadParams.from_host(hw, device="cuda")
    x = configs.hidden_states(c, device="cuda")
    pd = torch.as_tensor(pos.astype(np.float32)).cuda()
    sv, sa = sigma_pair(c.sigma_v)
    ws = torch.empty(api.workspace_size(dims, n), dtype=torch.uint8, device="cuda")
    ts, slot = O.plan_timesteps(sv, sa, segs)
    rows_of = O.token_rows(segs, slot, n)
    sample = _sample_rows(segs, n)
    pos64 = f64(pos)

    def check_block(i, x_in):
        """GPU block i on x_in (in place on a copy) against the oracle's block i
        on the same x_in."""
        x_out = x_in.clone()
        api.block_forward(dims, blocks[i], x_out, segs, pd, sv, sa, ws)
        api.device_status()
        p = _host_weights(c, i, blocks[i])
        mods = O.block_mods(p["adaln_w"], p["adaln_b"], p["adaln_table"], ts, c.hidden)
        xin64 = f64(x_in)
        ref = O.block_forward(p, xin64, mods, rows_of, pos64, c.dims(), sample_rows=sample)
        got = x_out[sample]
        assert_close(got, ref, what=f"block {i} x_out rows")
        assert_close(f64(got) - xin64[sample], ref - xin64[sample], what=f"block {i} delta rows")
        return x_out

    # blocks 0 .. 49 on the GPU, stopping at 0, 24 and 49 for the oracle
    xi = x.clone()
    done = 0
    for i in (0, 24, 49):
        if i > done:
            api.stack_forward(dims, blocks[done:i], None, xi, segs, pd, sv, sa, None, None, ws)
        xi = check_block(i, xi)
        done = i + 1
    assert done == c.n_blocks
    # the heads on the GPU's final hidden states
    vs = [s for s in segs if s[2] == 0][-1]
    a_segs = [s for s in segs if s[2] == 2]
    ov = torch.full((vs[1] - vs[0], 128), float("nan"), device="cuda")
    oa = torch.full((a_segs[-1][1] - a_segs[-1][0], 128), float("nan"), device="cuda") if a_segs else None
    api.stack_forward(dims, [], heads, xi, segs, pd, sv, sa, ov, oa, ws)
    api.device_status()
    fm = O.final_mods(f64(hw["adaln_w"]), f64(hw["adaln_b"]), f64(hw["adaln_table"]), ts, c.hidden)
    streams = [(vs, "video", ov)] + ([(a_segs[-1], "audio", oa)] if a_segs else [])
    for (seg, key, out) in streams:
        r = np.unique(np.concatenate([np.linspace(seg[0], seg[1] - 1, 9).astype(int),
                                      [seg[1] - 1, seg[1] - 2]]))
        ref = O.heads_forward(f64(xi[r]), f64(hw["final_norm"]), fm[slot[seg[3]]],
                              f64(hw[f"w_{key}"]), f64(hw[f"b_{key}"]), c.eps)
        assert_close(out[r - seg[0]], ref, what=f"{key} head rows after 50 blocks", rel=BF16_STORE_REL)


@pytest.mark.parametrize("act", [torch.float32, torch.bfloat16])
def test_tiny_shape_fifty_block_chain(cuda_ok, act):
    c = configs.TINY
    L = O.layout_t2va(c.text_len, c.latent_t, c.lat_h, c.lat_w, c.audio_t)
    segs, pos, n = L["segments"], L["pos"], L["seq_len"]
    assert n == 64
    nb = 50
    ws_ = [configs.block_weights(c, b, wdtype=act) for b in range(nb)]
    x = configs.hidden_states(c)
    sv, sa = sigma_pair(c.sigma_v)
    dims_c = api.make_dims(c.hidden, c.heads, c.head_dim, c.ffn, act_dtype=act)
    bp = [api.BlockParams.from_host(dims_c, w) for w in ws_]
    xd = x.cuda().clone()
    pd = torch.as_tensor(pos.astype(np.float32)).cuda()
    ws = torch.empty(api.workspace_size(dims_c, n), dtype=torch.uint8, device="cuda")
    api.stack_forward(dims_c, bp, None, xd, segs, pd, sv, sa, None, None, ws)
    api.device_status()
    ts, slot = O.plan_timesteps(sv, sa, segs)
    rows = O.token_rows(segs, slot, n)
    h = f64(x)
    for w in ws_:
        p = {k: f64(v) for k, v in w.items()}
        mods = O.block_mods(p["adaln_w"], p["adaln_b"], p["adaln_table"], ts, c.hidden)
        h = O.block_forward(p, h, mods, rows, pos, c.dims())
    if act == torch.float32:
        assert_close(xd, h, TF32_MAXABS, TF32_COS, "50-block chain x (fp32 storage)")
        assert_close(xd.cpu().double() - x.double(), h - f64(x), TF32_MAXABS, TF32_COS,
                     "50-block chain delta (fp32 storage)")
    else:
        assert_close(xd, h, what="50-block chain x (bf16 storage)")
        assert_close(xd.cpu().double() - x.double(), h - f64(x), what="50-block chain delta (bf16 storage)")


@pytest.mark.parametrize("n_blocks,layout", [(5, (2, 1, 4, 4, 1)), (7, (20, 3, 16, 20, 20))])
def test_stack_modulation_batches(cuda_ok, n_blocks, layout):
    # The stack evaluates its blocks' modulation in batches placed in the
    # head-scratch region: 8 tokens leave no room there (one block at a time
    # through the block's own modulation region), 300 tokens hold four
    # blocks' rows (batches of four and three).  Both against the oracle.
    from gpu_common import small_block_weights, small_dims, t2va
    dims_o, dims_c = small_dims()
    segs, pos = t2va(*layout)
    n = int(pos.shape[0])
    ws_ = [small_block_weights(70 + b, 256, 2, 128, 512) for b in range(n_blocks)]
    x = configs.synth.normal((n, 256), 83, 1.0)
    sv, sa = sigma_pair(0.5)
    bp = [api.BlockParams.from_host(dims_c, w) for w in ws_]
    xd = x.cuda().clone()
    pd = torch.as_tensor(np.asarray(pos, np.float32)).cuda()
    ws = torch.empty(api.workspace_size(dims_c, n), dtype=torch.uint8, device="cuda")
    api.stack_forward(dims_c, bp, None, xd, segs, pd, sv, sa, None, None, ws)
    api.device_status()
    ts, slot = O.plan_timesteps(sv, sa, segs)
    rows = O.token_rows(segs, slot, n)
    h = f64(x)
    for w in ws_:
        p = {k: f64(v) for k, v in w.items()}
        h = O.block_forward(p, h, O.block_mods(p["adaln_w"], p["adaln_b"], p["adaln_table"], ts, 256), rows,
                            f64(pos), dims_o)
    assert_close(xd, h, what=f"{n_blocks}-block stack x")
    assert_close(xd.cpu().double() - x.double(), h - f64(x), what=f"{n_blocks}-block stack delta")
