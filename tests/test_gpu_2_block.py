"""GPU parity of the whole modulated block (and its stack / heads) against
the oracle, through mmh3_block_forward / mmh3_stack_forward: the output, the
block delta (x_out - x_in) and every intermediate the workspace holds
(xn1, post-rotation q and k, v, attn, xn2, act)."""

import pytest

from gpu_common import (BF16_COS, BF16_MAXABS, BF16_STORE_REL, TF32_COS, TF32_MAXABS, TF32_STORE_REL, O,
                        api, assert_close,
                        configs, f64, heads_split, np, oracle_block, run_block, sigma_pair,
                        small_block_weights, small_dims, t2va, torch)

pytestmark = pytest.mark.gpu


def _check_block(dims_o, dims_c, w, x, segs, pos, sv, sa, bars, modulated=True):
    keep = {}
    ref, mods, rows = oracle_block(w, x, segs, pos, sv, sa, dims_o, keep=keep, modulated=modulated)
    xg, reg = run_block(dims_c, w, x, segs, pos, sv, sa, modulated=modulated)
    maxabs, cos, rel = bars
    H, nh, hd = dims_o["hidden"], dims_o["heads"], dims_o["head_dim"]
    # intermediates in path order, so the first failure names the step
    assert_close(reg["xn1"], keep["xn1"], maxabs, cos, "xn1", rel)
    q, k, v = heads_split(reg["qkv"], nh, hd)
    assert_close(q, keep["q"], maxabs, cos, "q after qk-norm + rotation", rel)
    assert_close(k, keep["k"], maxabs, cos, "k after qk-norm + rotation", rel)
    assert_close(v, keep["v"], maxabs, cos, "v", rel)
    assert_close(reg["attn"], keep["attn"], maxabs, cos, "attn", rel)
    assert_close(reg["xn2"], keep["xn2"], maxabs, cos, "xn2", rel)
    assert_close(reg["act"], keep["act"], maxabs, cos, "SwiGLU act", rel)
    assert_close(xg, ref, maxabs, cos, "x_out")
    assert_close(xg.cpu().double() - x.double(), ref - f64(x), maxabs, cos, "block delta")
    return xg


@pytest.mark.parametrize("layout,sigma_v", [((20, 3, 16, 20, 20), 0.5), ((5, 1, 4, 4, 3), 0.3),
                                            ((130, 2, 16, 16, 64), 1.0)])
def test_block_small_bf16(cuda_ok, layout, sigma_v):
    dims_o, dims_c = small_dims()
    segs, pos = t2va(*layout)
    n = int(pos.shape[0])
    w = small_block_weights(31, 256, 2, 128, 512)
    x = configs.synth.normal((n, 256), 77, 1.0)
    sv, sa = sigma_pair(sigma_v)
    _check_block(dims_o, dims_c, w, x, segs, pos, sv, sa, (BF16_MAXABS, BF16_COS, BF16_STORE_REL))


def test_block_zero_gates_is_exact_identity(cuda_ok):
    dims_o, dims_c = small_dims()
    segs, pos = t2va(20, 3, 16, 20, 20)
    n = int(pos.shape[0])
    w = small_block_weights(32, 256, 2, 128, 512)
    H = 256
    for e in (2, 5):
        for r in range(6):
            lo = r * 6 * H + e * H
            w["adaln_w"][lo:lo + H] = 0
            w["adaln_b"][lo:lo + H] = 0
    x = configs.synth.normal((n, H), 78, 1.0)
    xg, _ = run_block(dims_c, w, x, segs, pos, *sigma_pair(0.5))
    assert torch.equal(xg.cpu(), x)


def test_block_unmodulated_refiner_form(cuda_ok):
    dims_o, dims_c = small_dims()
    n = 150
    w = small_block_weights(33, 256, 2, 128, 512)
    x = configs.synth.normal((n, 256), 79, 1.0)
    segs = [(0, n, 1, 0)]
    _check_block(dims_o, dims_c, w, x, segs, None, 0.5, 0.2, (BF16_MAXABS, BF16_COS, BF16_STORE_REL), modulated=False)


def test_block_deterministic(cuda_ok):
    dims_o, dims_c = small_dims()
    segs, pos = t2va(20, 3, 16, 20, 20)
    w = small_block_weights(34, 256, 2, 128, 512)
    x = configs.synth.normal((int(pos.shape[0]), 256), 80, 1.0)
    a, _ = run_block(dims_c, w, x, segs, pos, *sigma_pair(0.5))
    b, _ = run_block(dims_c, w, x, segs, pos, *sigma_pair(0.5))
    assert torch.equal(a, b)


def test_tiny_workload_fp32(cuda_ok):
    c = configs.TINY
    segs, pos = t2va(c.text_len, c.latent_t, c.lat_h, c.lat_w, c.audio_t)
    assert pos.shape[0] == 64
    w = configs.block_weights(c, 0)
    x = configs.hidden_states(c)
    dims_c = api.make_dims(c.hidden, c.heads, c.head_dim, c.ffn, act_dtype=torch.float32)
    _check_block(c.dims(), dims_c, w, x, segs, pos, *sigma_pair(c.sigma_v), (TF32_MAXABS, TF32_COS, TF32_STORE_REL))


def test_tiny_workload_bf16(cuda_ok):
    c = configs.TINY
    segs, pos = t2va(c.text_len, c.latent_t, c.lat_h, c.lat_w, c.audio_t)
    w = configs.block_weights(c, 0, wdtype=torch.bfloat16)
    x = configs.hidden_states(c)
    dims_c = api.make_dims(c.hidden, c.heads, c.head_dim, c.ffn, act_dtype=torch.bfloat16)
    _check_block(c.dims(), dims_c, w, x, segs, pos, *sigma_pair(c.sigma_v), (BF16_MAXABS, BF16_COS, BF16_STORE_REL))


def test_block_workload_full_size_sampled_rows(cuda_ok):
    """The 13 248-token MiniMax-H3 block in the launch configuration the bench
    times; the oracle computes k and v for every token and the rest for a
    sample of rows spanning text, audio, video and the ragged last tile."""
    c = configs.BLOCK
    segs, pos = t2va(c.text_len, c.latent_t, c.lat_h, c.lat_w, c.audio_t)
    n = int(pos.shape[0])
    assert n == 13248
    w = configs.block_weights(c, 0)
    x = configs.hidden_states(c)
    sv, sa = sigma_pair(c.sigma_v)
    dims_c = api.make_dims(c.hidden, c.heads, c.head_dim, c.ffn)
    xg, reg = run_block(dims_c, w, x, segs, pos, sv, sa)
    sample = [0, 1, 255, 256, 511, 767, 768, 4000, 9000, 13119, 13120, 13200, 13247]
    keep = {}
    ref, _, _ = oracle_block(w, x, segs, pos, sv, sa, c.dims(), sample_rows=sample, keep=keep)
    assert_close(xg[sample], ref, what="x_out rows")
    assert_close(xg[sample].cpu().double() - x[sample].double(), ref - f64(x[sample]), what="delta rows")
    q, k, v = heads_split(reg["qkv"][sample], c.heads, c.head_dim)
    assert_close(reg["xn1"][sample], keep["xn1"], what="xn1 rows", rel=BF16_STORE_REL)
    assert_close(q, keep["q"], what="q rows", rel=BF16_STORE_REL)
    assert_close(k, keep["k"], what="k rows", rel=BF16_STORE_REL)
    assert_close(reg["attn"][sample], keep["attn"], what="attn rows", rel=BF16_STORE_REL)
    assert_close(reg["xn2"][sample], keep["xn2"], what="xn2 rows", rel=BF16_STORE_REL)
    assert_close(reg["act"][sample], keep["act"], what="act rows", rel=BF16_STORE_REL)


@pytest.mark.parametrize("layout", [(16, 2, 20, 20, 20), (17, 2, 20, 20, 20), (16, 2, 8, 82, 20),
                                    (17, 2, 24, 38, 20)])
def test_block_pair_tile_boundaries(cuda_ok, layout):
    # n = 256, 257, 384, 513: one exact 256-row pair tile; a second pair tile
    # whose upper CTA holds no row (its loads and stores are skipped); a
    # second tile whose lower CTA is full; a single valid row in the last tile
    dims_o, dims_c = small_dims()
    segs, pos = t2va(*layout)
    n = int(pos.shape[0])
    w = small_block_weights(35, 256, 2, 128, 512)
    x = configs.synth.normal((n, 256), 85, 1.0)
    sv, sa = sigma_pair(0.5)
    _check_block(dims_o, dims_c, w, x, segs, pos, sv, sa, (BF16_MAXABS, BF16_COS, BF16_STORE_REL))


def test_block_hidden_128_half_empty_tiles(cuda_ok):
    # hidden 128: the out and fc2 projections (N = 128) have one 256-wide
    # column tile per pair tile, whose upper CTA's half of B lies wholly
    # beyond N (zero-filled, its columns skipped by the epilogue)
    dims_o, dims_c = small_dims(hidden=128, heads=1, head_dim=128, ffn=256)
    segs, pos = t2va(20, 3, 16, 20, 20)
    n = int(pos.shape[0])
    w = small_block_weights(39, 128, 1, 128, 256)
    x = configs.synth.normal((n, 128), 86, 1.0)
    _check_block(dims_o, dims_c, w, x, segs, pos, *sigma_pair(0.5), (BF16_MAXABS, BF16_COS, BF16_STORE_REL))


def test_block_full_hidden_short_sequence(cuda_ok):
    # the block's own sizes (hidden 2688, 21 x 128 heads, SwiGLU 10752) at
    # 300 tokens: two pair-tile rows (the second one partly beyond n), 10.5
    # column tiles for out and fc2, 84 for fc1, 31.5 for qkv, attention in
    # three key tiles; sampled rows against the oracle
    c = configs.BLOCK
    segs, pos = t2va(20, 3, 16, 20, 20)
    n = int(pos.shape[0])
    assert 257 <= n <= 512
    w = configs.block_weights(c, 0)
    x = configs.hidden_states(c, n)
    sv, sa = sigma_pair(c.sigma_v)
    dims_c = api.make_dims(c.hidden, c.heads, c.head_dim, c.ffn)
    xg, reg = run_block(dims_c, w, x, segs, pos, sv, sa)
    sample = [0, 1, 100, 255, 256, n - 1]
    keep = {}
    ref, _, _ = oracle_block(w, x, segs, pos, sv, sa, c.dims(), sample_rows=sample, keep=keep)
    assert_close(reg["attn"][sample], keep["attn"], what="attn rows", rel=BF16_STORE_REL)
    assert_close(xg[sample], ref, what="x_out rows")
    assert_close(xg[sample].cpu().double() - x[sample].double(), ref - f64(x[sample]), what="delta rows")


def test_block_forward_host_pipelined_matches_device_calls(cuda_ok):
    # seven calls rotating over the slots with different inputs: each result
    # is the device block's on the same input, bit for bit
    dims_o, dims_c = small_dims()
    segs, pos = t2va(20, 3, 16, 20, 20)
    n = int(pos.shape[0])
    w = small_block_weights(36, 256, 2, 128, 512)
    params = api.BlockParams.from_host(dims_c, w)
    sv, sa = sigma_pair(0.5)
    ws = torch.empty(api.workspace_size(dims_c, n), dtype=torch.uint8, device="cuda")
    pos_h = torch.as_tensor(np.asarray(pos, np.float32)).pin_memory()
    calls = 7
    xs = [configs.synth.normal((n, 256), 95 + k, 1.0).pin_memory() for k in range(calls)]
    outs = [torch.empty_like(x).pin_memory() for x in xs]
    x_dev = [torch.empty((n, 256), device="cuda") for _ in range(api.HOST_SLOTS)]
    p_dev = [torch.empty((n, 3), device="cuda") for _ in range(api.HOST_SLOTS)]
    cin, cout = torch.cuda.Stream(), torch.cuda.Stream()
    for k in range(calls):
        slot = k % api.HOST_SLOTS
        api.block_forward_host(dims_c, params, xs[k], outs[k], segs, pos_h, sv, sa, slot, x_dev[slot],
                               p_dev[slot], ws, cin, cout)
    cout.synchronize()
    torch.cuda.synchronize()
    api.device_status()
    pd = pos_h.cuda()
    for k in range(calls):
        ref = xs[k].cuda()
        api.block_forward(dims_c, params, ref, segs, pd, sv, sa, ws)
        assert torch.equal(outs[k], ref.cpu()), f"call {k}"


def test_launch_count_of_one_block(cuda_ok):
    # prologue (adaLN curve + rotation table), 2 x norm/modulate, 4 GEMMs,
    # attention: 8 kernels (attention adds a merge launch when its last wave
    # is split)
    dims_o, dims_c = small_dims()
    segs, pos = t2va(20, 3, 16, 20, 20)
    n = int(pos.shape[0])
    w = small_block_weights(37, 256, 2, 128, 512)
    x = configs.synth.normal((n, 256), 97, 1.0)
    params = api.BlockParams.from_host(dims_c, w)
    xd = x.cuda()
    pd = torch.as_tensor(np.asarray(pos, np.float32)).cuda()
    ws = torch.empty(api.workspace_size(dims_c, n), dtype=torch.uint8, device="cuda")
    c0 = api.launch_count()
    api.block_forward(dims_c, params, xd, segs, pd, *sigma_pair(0.5), ws)
    assert api.launch_count() - c0 == 8


def test_block_caller_modulation_replaces_the_adaln_curve(cuda_ok):
    # mods_or_null: the oracle's modulation at timesteps other than the
    # plan's (so the block's own curve would give different rows) is passed
    # in, with the adaLN weights left out of the weight struct; the block
    # must match the oracle block run on exactly those rows.
    dims_o, dims_c = small_dims()
    segs, pos = t2va(20, 3, 16, 20, 20)
    n = int(pos.shape[0])
    w = small_block_weights(35, 256, 2, 128, 512)
    x = configs.synth.normal((n, 256), 81, 1.0)
    sv, sa = sigma_pair(0.5)
    ts, slot = O.plan_timesteps(sv, sa, segs)
    rows = O.token_rows(segs, slot, n)
    mods = O.block_mods(f64(w["adaln_w"]), f64(w["adaln_b"]), f64(w["adaln_table"]), [0.15, 0.85], 256)
    ref = O.block_forward({k: f64(v) for k, v in w.items()}, f64(x), mods, rows, f64(pos), dims_o)
    params = api.BlockParams.from_host(dims_c, {k: v for k, v in w.items() if not k.startswith("adaln")})
    xd = x.cuda().clone()
    pd = torch.as_tensor(np.asarray(pos, dtype=np.float32)).cuda()
    ws = torch.empty(api.workspace_size(dims_c, n), dtype=torch.uint8, device="cuda")
    md = torch.as_tensor(mods.astype(np.float32)).cuda()
    api.block_forward(dims_c, params, xd, segs, pd, sv, sa, ws, mods=md)
    assert api.status_sync() == 0
    assert_close(xd, ref, what="x_out with caller modulation")
    assert_close(xd.cpu().double() - x.double(), ref - f64(x), what="block delta with caller modulation")
    # the block's own curve gives other rows: its delta would fail the bar
    own, _, _ = oracle_block(w, x, segs, pos, sv, sa, dims_o)
    from gpu_common import cosine
    assert cosine(own - f64(x), ref - f64(x)) < BF16_COS


def _graph_vs_eager(dims_c, w, segs, pos, sv, sa, xs, launches):
    """One block forward captured in a CUDA graph, then replayed on each input
    of `xs` (copied into the captured x): every replay equals the eager call on
    the same input, bit for bit, and the capture holds `launches` kernels."""
    n, H = xs[0].shape
    params = api.BlockParams.from_host(dims_c, w, device="cuda")
    pd = torch.as_tensor(np.asarray(pos, np.float32)).cuda()
    ws = torch.empty(api.workspace_size(dims_c, n), dtype=torch.uint8, device="cuda")
    xg = xs[0].cuda().clone()
    api.block_forward(dims_c, params, xg, segs, pd, sv, sa, ws)  # first-use set-up outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    c0 = api.launch_count()
    with torch.cuda.graph(g):
        api.block_forward(dims_c, params, xg, segs, pd, sv, sa, ws)
    assert api.launch_count() - c0 == launches
    for k, x in enumerate(xs):
        xg.copy_(x.cuda())
        g.replay()
        ref = x.cuda().clone()
        api.block_forward(dims_c, params, ref, segs, pd, sv, sa, ws)
        torch.cuda.synchronize()
        assert torch.equal(xg, ref), f"replay {k}"
    g.reset()
    assert api.status_sync() == 0


def test_block_graph_replay_matches_eager(cuda_ok):
    dims_o, dims_c = small_dims()
    segs, pos = t2va(20, 3, 16, 20, 20)
    n = int(pos.shape[0])
    w = small_block_weights(38, 256, 2, 128, 512)
    xs = [configs.synth.normal((n, 256), 110 + k, 1.0) for k in range(3)]
    _graph_vs_eager(dims_c, w, segs, pos, *sigma_pair(0.5), xs, 8)


def test_block_workload_graph_replay_matches_eager(cuda_ok):
    # the bench's launch configuration: the attention's last wave is split,
    # so the capture holds the merge launch as well
    c = configs.BLOCK
    segs, pos = t2va(c.text_len, c.latent_t, c.lat_h, c.lat_w, c.audio_t)
    n = int(pos.shape[0])
    w = configs.block_weights(c, 0, device="cuda")
    x0 = configs.hidden_states(c, device="cuda")
    xs = [x0, x0 * 0.5]
    dims_c = api.make_dims(c.hidden, c.heads, c.head_dim, c.ffn)
    _graph_vs_eager(dims_c, w, segs, pos, *sigma_pair(c.sigma_v), xs, 9)
