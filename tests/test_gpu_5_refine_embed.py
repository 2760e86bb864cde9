"""GPU parity of the token refiner, the embed (patchify / audio packing and
the patch projections) and the output unpacking against the oracle, through
mmh3_refine_text, mmh3_patch_embed, mmh3_embed, mmh3_unpatchify_video and
mmh3_unpack_audio.

The embed inputs are made bf16-representable on the host, so the kernel's
rounding of the patch rows to the projection's operand type is exact; what
is left is fp32 accumulation over K <= 64 terms, hence the tight bars."""

import pytest

from gpu_common import (BF16_COS, BF16_MAXABS, TF32_COS, TF32_MAXABS, O, api, assert_close,
                        configs, f64, np, oracle_params, small_block_weights, small_dims, torch)

pytestmark = pytest.mark.gpu

EXACT_ACC = 1e-4        # fp32 accumulation of <= 192 exact products of O(1) terms


def _bf16_exact(shape, seed, std=1.0):
    return configs.synth.normal(shape, seed, std).to(torch.bfloat16).float()


def _refine_case(act, hidden, heads, head_dim, ffn, n, text_dim, n_blocks):
    dims_o, dims_c = small_dims(hidden, heads, head_dim, ffn, act=act)
    states = configs.synth.normal((n, text_dim), 501, 1.0).to(act)
    cond_w = configs.synth.normal((hidden, text_dim), 502, text_dim ** -0.5).to(act)
    cond_b = configs.synth.normal((hidden,), 503, 0.1)
    norm = 1.0 + configs.synth.normal((hidden,), 504, 0.1)
    blocks = [small_block_weights(510 + i, hidden, heads, head_dim, ffn, wdtype=act)
              for i in range(n_blocks)]
    final_eps = 1e-6
    ref = O.refine_text(f64(states), f64(cond_w), f64(cond_b), [oracle_params(w) for w in blocks],
                        f64(norm), dims_o, final_eps)
    params = [api.BlockParams.from_host(dims_c, w) for w in blocks]
    out = torch.empty((n, hidden), dtype=torch.float32, device="cuda")
    ws = torch.empty(api.refine_workspace_size(dims_c, n), dtype=torch.uint8, device="cuda")
    api.refine_text(dims_c, states.cuda(), cond_w.cuda(), cond_b.cuda(), params, norm.cuda(),
                    final_eps, out, ws)
    api.device_status()
    return out, ref


def test_refine_projection_and_norm_only(cuda_ok):
    # no refiner blocks: out = RMSNorm(states W^T + b); the products of bf16
    # operands are exact in fp32, so only accumulation order differs
    out, ref = _refine_case(torch.bfloat16, 256, 2, 128, 512, 77, 192, 0)
    assert_close(out, ref, EXACT_ACC, 0.9999999, "refine (no blocks)")


def test_refine_two_blocks_bf16(cuda_ok):
    out, ref = _refine_case(torch.bfloat16, 256, 2, 128, 512, 77, 192, 2)
    assert_close(out, ref, BF16_MAXABS, BF16_COS, "refine (2 blocks, bf16)")


def test_refine_one_block_fp32(cuda_ok):
    out, ref = _refine_case(torch.float32, 128, 2, 64, 256, 45, 96, 1)
    assert_close(out, ref, TF32_MAXABS, TF32_COS, "refine (1 block, fp32)")


@pytest.mark.parametrize("C,T,lh,lw", [(16, 3, 10, 14), (4, 1, 2, 2), (2, 5, 32, 34)])
def test_patch_embed_video(cuda_ok, C, T, lh, lw):
    H = 256
    _, dims_c = small_dims(H, 2, 128, 512)
    lat = _bf16_exact((C, T, lh, lw), 601 + C)
    w = configs.synth.normal((H, 4 * C), 602, (4 * C) ** -0.5).to(torch.bfloat16)
    b = configs.synth.normal((H,), 603, 0.1)
    rows = T * (lh // 2) * (lw // 2)
    x = torch.full((rows + 1, H), 7.0, device="cuda")          # one guard row past the end
    ws = torch.empty(api.patch_embed_workspace_size(dims_c, api.MMH3_STREAM_VIDEO, lat.shape),
                     dtype=torch.uint8, device="cuda")
    api.patch_embed(dims_c, api.MMH3_STREAM_VIDEO, lat.cuda(), w.cuda(), b.cuda(), x[:rows], ws)
    ref = O.patchify_video(f64(lat)) @ f64(w).T + f64(b)
    assert_close(x[:rows], ref, EXACT_ACC, 0.9999999, "video patch embed")
    assert (x[rows] == 7.0).all(), "patch embed wrote past its rows"


@pytest.mark.parametrize("C,T", [(24, 37), (8, 64), (64, 3)])
def test_patch_embed_audio(cuda_ok, C, T):
    H = 128
    _, dims_c = small_dims(H, 1, 128, 256)
    lat = _bf16_exact((C, 2, T), 611 + C)
    w = configs.synth.normal((H, C), 612, C ** -0.5).to(torch.bfloat16)
    b = configs.synth.normal((H,), 613, 0.1)
    x = torch.empty((2 * T, H), device="cuda")
    ws = torch.empty(api.patch_embed_workspace_size(dims_c, api.MMH3_STREAM_AUDIO, lat.shape),
                     dtype=torch.uint8, device="cuda")
    api.patch_embed(dims_c, api.MMH3_STREAM_AUDIO, lat.cuda(), w.cuda(), b.cuda(), x, ws)
    ref = O.pack_audio(f64(lat)) @ f64(w).T + f64(b)
    assert_close(x, ref, EXACT_ACC, 0.9999999, "audio patch embed")


def _embed_weights(H, Cv, Ca):
    wv = configs.synth.normal((H, 4 * Cv), 621, (4 * Cv) ** -0.5).to(torch.bfloat16)
    bv = configs.synth.normal((H,), 622, 0.1)
    wa = configs.synth.normal((H, Ca), 623, Ca ** -0.5).to(torch.bfloat16)
    ba = configs.synth.normal((H,), 624, 0.1)
    return wv, bv, wa, ba


def test_embed_t2va_layout(cuda_ok):
    H, Cv, Ca = 128, 4, 8
    _, dims_c = small_dims(H, 1, 128, 256)
    L = O.layout_t2va(5, 2, 6, 8, 7)
    segs, n = L["segments"], L["seq_len"]
    text = configs.synth.normal((5, H), 631, 1.0)
    video = _bf16_exact((Cv, 2, 6, 8), 632)
    audio = _bf16_exact((Ca, 2, 7), 633)
    wv, bv, wa, ba = _embed_weights(H, Cv, Ca)
    ref = O.embed(L, f64(text), f64(video), f64(audio), f64(wv), f64(bv), f64(wa), f64(ba))
    x = torch.full((n, H), float("nan"), device="cuda")
    d = [t.cuda() for t in (text, video, audio, wv, bv, wa, ba)]
    ws = torch.empty(api.embed_workspace_size(dims_c, d[0], d[1], d[2]), dtype=torch.uint8,
                     device="cuda")
    api.embed(dims_c, segs, n, d[0], d[1], d[2], d[3], d[4], d[5], d[6], x, ws)
    assert torch.equal(x[:5].cpu(), text), "text rows are a copy"
    assert_close(x, ref, EXACT_ACC, 0.9999999, "embed (t2va)")


def test_embed_with_condition_frames(cuda_ok):
    # [text 3 | cond frame | cond frame | target video, 2 frames | audio 2x5]
    H, Cv, Ca, lh, lw = 128, 2, 16, 4, 6
    _, dims_c = small_dims(H, 1, 128, 256)
    fr = (lh // 2) * (lw // 2)
    segs, a = [(0, 3, 1, 0)], 3
    for rows, tag, clock in ((fr, 0, 0), (fr, 0, 0), (2 * fr, 0, 0), (2 * 5, 2, 1)):
        segs.append((a, a + rows, tag, clock))
        a += rows
    n = a
    L = {"seq_len": n, "segments": segs}
    text = configs.synth.normal((3, H), 641, 1.0)
    video = _bf16_exact((Cv, 2, lh, lw), 642)
    cond = [_bf16_exact((Cv, 1, lh, lw), 643 + i) for i in range(2)]
    audio = _bf16_exact((Ca, 2, 5), 645)
    wv, bv, wa, ba = _embed_weights(H, Cv, Ca)
    ref = O.embed(L, f64(text), f64(video), f64(audio), f64(wv), f64(bv), f64(wa), f64(ba),
                  cond=[f64(z) for z in cond])
    x = torch.full((n, H), float("nan"), device="cuda")
    d = [t.cuda() for t in (text, video, audio, wv, bv, wa, ba)]
    dc = [z.cuda() for z in cond]
    ws = torch.empty(api.embed_workspace_size(dims_c, d[0], d[1], d[2], dc), dtype=torch.uint8,
                     device="cuda")
    api.embed(dims_c, segs, n, d[0], d[1], d[2], d[3], d[4], d[5], d[6], x, ws, cond=dc)
    assert_close(x, ref, EXACT_ACC, 0.9999999, "embed (condition frames)")


def test_unpatchify_and_unpack_are_the_oracle_inverses(cuda_ok):
    C, T, lh, lw = 3, 4, 6, 10
    rows = configs.synth.normal((T * (lh // 2) * (lw // 2), 4 * C), 651, 1.0)
    out = torch.empty((C, T, lh, lw), device="cuda")
    api.unpatchify_video(rows.cuda(), C, T, lh, lw, out)
    assert torch.equal(out.cpu(), torch.as_tensor(O.unpatchify_video(rows.numpy(), C, T, lh, lw)))
    Ca, Ta = 5, 9
    arows = configs.synth.normal((2 * Ta, Ca), 652, 1.0)
    aout = torch.empty((Ca, 2, Ta), device="cuda")
    api.unpack_audio(arows.cuda(), Ca, Ta, aout)
    assert torch.equal(aout.cpu(), torch.as_tensor(O.unpack_audio(arows.numpy(), Ca, Ta)))


def test_denoise_forward_end_to_end(cuda_ok):
    # embed -> 2 blocks -> heads -> unpatchify / unpack through one call
    dims_o, dims_c = small_dims()
    H, Cv, Ca = 256, 8, 32
    L = O.layout_t2va(8, 2, 8, 12, 6)
    segs, n = L["segments"], L["seq_len"]
    text = configs.synth.normal((8, H), 661, 1.0)
    video = _bf16_exact((Cv, 2, 8, 12), 662)
    audio = _bf16_exact((Ca, 2, 6), 663)
    ew = _embed_weights(H, Cv, Ca)
    blocks = [small_block_weights(670 + i, H, 2, 128, 512) for i in range(2)]
    cfg = configs.DitConfig("fwd", 68, hidden=H, heads=2, head_dim=128, ffn=512, text_len=1,
                            heads_out=32)
    heads = configs.head_weights(cfg)
    heads["w_audio"] = configs.synth.normal((Ca, H), 664, 0.02).to(torch.bfloat16)
    heads["b_audio"] = configs.synth.normal((Ca,), 665, 0.02)
    sv, sa = 0.5, O.time_shift_sigma(0.5, 12.0, 3.0)
    rv, ra = O.denoise_forward(L, f64(text), f64(video), f64(audio), tuple(f64(t) for t in ew),
                               [oracle_params(w) for w in blocks], oracle_params(heads), sv, sa,
                               dims_o)
    bp = [api.BlockParams.from_host(dims_c, w) for w in blocks]
    hp = api.HeadParams.from_host(heads)
    d = [t.cuda() for t in (text, video, audio)]
    pos = torch.as_tensor(np.asarray(L["pos"], np.float32)).cuda()
    x = torch.empty((n, H), device="cuda")
    vo = torch.full(video.shape, float("nan"), device="cuda")
    ao = torch.full(audio.shape, float("nan"), device="cuda")
    ws = torch.empty(api.forward_workspace_size(dims_c, n, *d), dtype=torch.uint8, device="cuda")
    api.forward(dims_c, segs, n, pos, sv, sa, *d, tuple(t.cuda() for t in ew), bp, hp, x, vo, ao,
                ws)
    api.device_status()
    assert_close(vo, rv, BF16_MAXABS, BF16_COS, "video velocity")
    assert_close(ao, ra, BF16_MAXABS, BF16_COS, "audio velocity")


def _graph_equals_eager(fn, outs):
    """fn() once eagerly, then captured in a CUDA graph and replayed; the
    replay's outputs equal the eager call's bit for bit."""
    fn()
    torch.cuda.synchronize()
    eager = [t.clone() for t in outs]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    for t in outs:
        t.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    g.reset()
    assert api.status_sync() == 0
    for a, b in zip(outs, eager):
        assert torch.equal(a, b)


def test_denoise_forward_graph_replay(cuda_ok):
    # mmh3_forward (embed, two blocks, heads, unpatchify / unpack) captured
    # in a CUDA graph
    dims_o, dims_c = small_dims()
    H, Cv, Ca = 256, 8, 32
    L = O.layout_t2va(8, 2, 8, 12, 6)
    segs, n = L["segments"], L["seq_len"]
    d = [configs.synth.normal((8, H), 681, 1.0).cuda(), _bf16_exact((Cv, 2, 8, 12), 682).cuda(),
         _bf16_exact((Ca, 2, 6), 683).cuda()]
    ew = tuple(t.cuda() for t in _embed_weights(H, Cv, Ca))
    bp = [api.BlockParams.from_host(dims_c, small_block_weights(690 + i, H, 2, 128, 512)) for i in range(2)]
    cfg = configs.DitConfig("fwdg", 69, hidden=H, heads=2, head_dim=128, ffn=512, text_len=1, heads_out=32)
    heads = configs.head_weights(cfg)
    heads["w_audio"] = configs.synth.normal((Ca, H), 684, 0.02).to(torch.bfloat16)
    heads["b_audio"] = configs.synth.normal((Ca,), 685, 0.02)
    hp = api.HeadParams.from_host(heads)
    pos = torch.as_tensor(np.asarray(L["pos"], np.float32)).cuda()
    x = torch.empty((n, H), device="cuda")
    vo = torch.empty(d[1].shape, device="cuda")
    ao = torch.empty(d[2].shape, device="cuda")
    ws = torch.empty(api.forward_workspace_size(dims_c, n, *d), dtype=torch.uint8, device="cuda")
    sv, sa = 0.5, O.time_shift_sigma(0.5, 12.0, 3.0)
    _graph_equals_eager(lambda: api.forward(dims_c, segs, n, pos, sv, sa, *d, ew, bp, hp, x, vo, ao, ws),
                        [x, vo, ao])


def test_refine_graph_replay(cuda_ok):
    dims_o, dims_c = small_dims()
    n, text_dim = 77, 384
    states = configs.synth.normal((n, text_dim), 701, 1.0).to(torch.bfloat16).cuda()
    cond_w = configs.synth.normal((256, text_dim), 702, text_dim ** -0.5).to(torch.bfloat16).cuda()
    cond_b = configs.synth.normal((256,), 703, 0.1).cuda()
    norm = (1.0 + configs.synth.normal((256,), 704, 0.1)).cuda()
    blocks = [api.BlockParams.from_host(dims_c, small_block_weights(710 + i, 256, 2, 128, 512)) for i in range(2)]
    out = torch.empty((n, 256), dtype=torch.float32, device="cuda")
    ws = torch.empty(api.refine_workspace_size(dims_c, n), dtype=torch.uint8, device="cuda")
    _graph_equals_eager(lambda: api.refine_text(dims_c, states, cond_w, cond_b, blocks, norm, 1e-6, out, ws),
                        [out])
