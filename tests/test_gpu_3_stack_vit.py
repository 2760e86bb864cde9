"""GPU parity of the stack with its output heads and of the SigLIP encoder
layer against the oracle."""

import pytest

from gpu_common import (BF16_COS, BF16_MAXABS, O, api, assert_close, configs, f64, math, np,
                        sigma_pair, small_block_weights, small_dims, t2va, torch)

pytestmark = pytest.mark.gpu


def _oracle_stack(blocks, heads, x, segs, pos, sv, sa, dims):
    n = x.shape[0]
    ts, slot = O.plan_timesteps(sv, sa, segs)
    rows = O.token_rows(segs, slot, n)
    h = f64(x)
    for w in blocks:
        mods = O.block_mods(f64(w["adaln_w"]), f64(w["adaln_b"]), f64(w["adaln_table"]), ts, dims["hidden"])
        h = O.block_forward({k: f64(v) for k, v in w.items()}, h, mods, rows, f64(pos), dims)
    outs = {}
    if heads is not None:
        fm = O.final_mods(f64(heads["adaln_w"]), f64(heads["adaln_b"]), f64(heads["adaln_table"]), ts,
                          dims["hidden"])
        for (a, b, tag, clock) in segs:
            if tag in (0, 2):
                key = "video" if tag == 0 else "audio"
                outs[key] = O.heads_forward(h[a:b], f64(heads["final_norm"]), fm[slot[clock]],
                                            f64(heads[f"w_{key}"]), f64(heads[f"b_{key}"]), dims["eps"])
    return h, outs


def _run_stack(dims_c, blocks, heads, x, segs, pos, sv, sa):
    bp = [api.BlockParams.from_host(dims_c, w) for w in blocks]
    hp = api.HeadParams.from_host(heads) if heads is not None else None
    xd = x.cuda().clone()
    pd = torch.as_tensor(np.asarray(pos, np.float32)).cuda()
    vseg = [s for s in segs if s[2] == 0][-1]
    aseg = [s for s in segs if s[2] == 2]
    ov = torch.full((vseg[1] - vseg[0], heads["w_video"].shape[0]), float("nan"), device="cuda") if heads else None
    oa = (torch.full((aseg[-1][1] - aseg[-1][0], heads["w_audio"].shape[0]), float("nan"), device="cuda")
          if heads and aseg else None)
    ws = torch.empty(api.workspace_size(dims_c, x.shape[0]), dtype=torch.uint8, device="cuda")
    api.stack_forward(dims_c, bp, hp, xd, segs, pd, sv, sa, ov, oa, ws)
    api.device_status()
    return xd, ov, oa


def _small_heads(seed, H, C=128):
    cfg = configs.DitConfig("h", seed, hidden=H, heads=2, head_dim=128, ffn=512, text_len=1, heads_out=C)
    return configs.head_weights(cfg)


def test_stack_small_with_heads(cuda_ok):
    dims_o, dims_c = small_dims()
    segs, pos = t2va(20, 3, 16, 20, 20)
    n = int(pos.shape[0])
    blocks = [small_block_weights(40 + i, 256, 2, 128, 512) for i in range(3)]
    heads = _small_heads(50, 256)
    x = configs.synth.normal((n, 256), 81, 1.0)
    sv, sa = sigma_pair(0.5)
    ref, outs = _oracle_stack(blocks, heads, x, segs, pos, sv, sa, dims_o)
    xg, ov, oa = _run_stack(dims_c, blocks, heads, x, segs, pos, sv, sa)
    assert_close(xg, ref, what="stack x")
    assert_close(xg.cpu().double() - x.double(), ref - f64(x), what="stack delta")
    assert_close(ov, outs["video"], what="video head")
    assert_close(oa, outs["audio"], what="audio head")


def test_stack_equals_repeated_blocks(cuda_ok):
    dims_o, dims_c = small_dims()
    segs, pos = t2va(20, 3, 16, 20, 20)
    n = int(pos.shape[0])
    blocks = [small_block_weights(60 + i, 256, 2, 128, 512) for i in range(3)]
    x = configs.synth.normal((n, 256), 82, 1.0)
    sv, sa = sigma_pair(0.3)
    ws = torch.empty(api.workspace_size(dims_c, n), dtype=torch.uint8, device="cuda")
    pd = torch.as_tensor(np.asarray(pos, np.float32)).cuda()
    bp = [api.BlockParams.from_host(dims_c, w) for w in blocks]
    x1 = x.cuda().clone()
    api.stack_forward(dims_c, bp, None, x1, segs, pd, sv, sa, None, None, ws)
    x2 = x.cuda().clone()
    for b in bp:
        api.block_forward(dims_c, b, x2, segs, pd, sv, sa, ws)
    api.device_status()
    assert torch.equal(x1, x2)


def _vit_small():
    cfg = configs.VitConfig("vs", 9, batch=2, seq=200, hidden=256, heads=4, head_dim=64, mlp=512)
    return cfg


def _oracle_vit(cfg, w, x, images=None):
    p = {k: f64(v) for k, v in w.items()}
    fq, fb = O.vit_fold_scale(p["wq"], p["bq"], cfg.head_dim)
    p["wqkv"] = np.concatenate([fq, p["wk"], p["wv"]])
    p["bqkv"] = np.concatenate([fb, p["bk"], p["bv"]])
    return O.vit_layer_forward(p, f64(x), cfg.batch, cfg.seq, cfg.dims(), images=images)


def _run_vit(cfg, w, x):
    d = api.vit_dims(cfg.hidden, cfg.heads, cfg.head_dim, cfg.mlp, cfg.ln_eps)
    params = api.VitParams.from_host(d, w)
    xd = x.cuda().clone()
    ws = torch.empty(api.vit_workspace_size(d, cfg.batch, cfg.seq), dtype=torch.uint8, device="cuda")
    api.vit_layer_forward(d, params, xd, cfg.batch, cfg.seq, ws)
    api.device_status()
    return xd


def test_vit_layer_small(cuda_ok):
    cfg = _vit_small()
    w = configs.vit_weights(cfg)
    x = configs.vit_inputs(cfg)
    ref = _oracle_vit(cfg, w, x)
    xg = _run_vit(cfg, w, x)
    assert_close(xg, ref, what="vit x")
    assert_close(xg.cpu().double() - x.double(), ref - f64(x), what="vit delta")


def test_vit_layer_full_size_sampled_images(cuda_ok):
    cfg = configs.SIGLIP
    w = configs.vit_weights(cfg)
    x = configs.vit_inputs(cfg)
    xg = _run_vit(cfg, w, x)
    for img in (0, 31):
        ref = _oracle_vit(cfg, w, x, images=[img])
        rows = slice(img * cfg.seq, (img + 1) * cfg.seq)
        assert_close(xg[rows], ref, what=f"image {img}")
        assert_close(xg[rows].cpu().double() - x[rows].double(), ref - f64(x[rows]), what=f"image {img} delta")


def _capture(fn):
    """fn() run once eagerly (first-use set-up), then captured in a CUDA graph."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


@pytest.mark.parametrize("act,heads,head_dim,ffn", [(torch.bfloat16, 2, 128, 512), (torch.float32, 4, 64, 1024)])
def test_stack_graph_replay_matches_eager(cuda_ok, act, heads, head_dim, ffn):
    # three blocks and the output heads in one captured graph (bf16 operands,
    # and fp32 storage with tf32 tensor-core GEMMs): a replay on a new input
    # equals the eager stack on it, bit for bit, heads included
    dims_o, dims_c = small_dims(heads=heads, head_dim=head_dim, ffn=ffn, act=act)
    segs, pos = t2va(20, 3, 16, 20, 20)
    n = int(pos.shape[0])
    bp = [api.BlockParams.from_host(dims_c, small_block_weights(70 + i, 256, heads, head_dim, ffn, wdtype=act))
          for i in range(3)]
    hp = api.HeadParams.from_host(_small_heads(71, 256))
    pd = torch.as_tensor(np.asarray(pos, np.float32)).cuda()
    vseg = [s for s in segs if s[2] == 0][-1]
    aseg = [s for s in segs if s[2] == 2][-1]
    ws = torch.empty(api.workspace_size(dims_c, n), dtype=torch.uint8, device="cuda")
    sv, sa = sigma_pair(0.5)

    def run(xd, ov, oa):
        api.stack_forward(dims_c, bp, hp, xd, segs, pd, sv, sa, ov, oa, ws)

    xg = configs.synth.normal((n, 256), 83, 1.0).cuda()
    ovg = torch.empty((vseg[1] - vseg[0], 128), device="cuda")
    oag = torch.empty((aseg[1] - aseg[0], 128), device="cuda")
    g = _capture(lambda: run(xg, ovg, oag))
    x_new = configs.synth.normal((n, 256), 84, 1.0).cuda()
    xg.copy_(x_new)
    g.replay()
    xe, ove, oae = x_new.clone(), torch.empty_like(ovg), torch.empty_like(oag)
    run(xe, ove, oae)
    torch.cuda.synchronize()
    g.reset()
    assert api.status_sync() == 0
    assert torch.equal(xg, xe) and torch.equal(ovg, ove) and torch.equal(oag, oae)


def test_vit_layer_graph_replay_matches_eager(cuda_ok):
    cfg = _vit_small()
    d = api.vit_dims(cfg.hidden, cfg.heads, cfg.head_dim, cfg.mlp, cfg.ln_eps)
    params = api.VitParams.from_host(d, configs.vit_weights(cfg))
    x = configs.vit_inputs(cfg).cuda()
    ws = torch.empty(api.vit_workspace_size(d, cfg.batch, cfg.seq), dtype=torch.uint8, device="cuda")
    xg = x.clone()
    g = _capture(lambda: api.vit_layer_forward(d, params, xg, cfg.batch, cfg.seq, ws))
    xg.copy_(x)
    g.replay()
    xe = x.clone()
    api.vit_layer_forward(d, params, xe, cfg.batch, cfg.seq, ws)
    torch.cuda.synchronize()
    g.reset()
    assert api.status_sync() == 0
    assert torch.equal(xg, xe)
