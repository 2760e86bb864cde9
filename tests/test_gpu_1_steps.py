"""GPU parity of the individual steps against the oracle, through the C ABI:
segment rows (exact), adaLN modulation (1e-4 relative), attention (bf16 bar)
on ragged, single-token, multi-sequence and large-score inputs, and the
bounded-wait error path."""

import pytest

from gpu_common import (BF16_COS, BF16_MAXABS, TF32_COS, TF32_MAXABS, O, api, assert_close,
                        configs, f64, math, np, sigma_pair, synth, torch)

pytestmark = pytest.mark.gpu


def _layout(name):
    c = configs.CONFIGS[name]
    if c.image_mode:
        return O.layout_image(c.text_len, c.ref_lat_h, c.ref_lat_w, c.lat_h, c.lat_w)
    return O.layout_t2va(c.text_len, c.latent_t, c.lat_h, c.lat_w, c.audio_t)


@pytest.mark.parametrize("name", ["tiny", "block", "stack", "image"])
@pytest.mark.parametrize("sigma_v", [0.3, 0.5, 1.0])
def test_rows_exact(cuda_ok, name, sigma_v):
    L = _layout(name)
    sv, sa = sigma_pair(sigma_v)
    ts, slot = O.plan_timesteps(sv, sa, L["segments"])
    ref = O.token_rows(L["segments"], slot, L["seq_len"])
    rows = torch.full((L["seq_len"],), -7, dtype=torch.int32, device="cuda")
    api.resolve_rows(L["segments"], L["seq_len"], sv, sa, rows)
    np.testing.assert_array_equal(rows.cpu().numpy(), ref)


@pytest.mark.parametrize("name", ["tiny", "block", "image"])
@pytest.mark.parametrize("sigma_v", [0.0, 0.3, 0.5, 0.97, 1.0])
def test_adaln_modulation(cuda_ok, name, sigma_v):
    c = configs.CONFIGS[name]
    L = _layout(name)
    w = configs.block_weights(c, 0, keys=("adaln_w", "adaln_b", "adaln_table"))
    sv, sa = sigma_pair(sigma_v)
    ts, _ = O.plan_timesteps(sv, sa, L["segments"])
    H = c.hidden
    ref = O.block_mods(f64(w["adaln_w"]), f64(w["adaln_b"]), f64(w["adaln_table"]), ts, H)
    out = torch.full((2 * 18 * H,), float("nan"), device="cuda")
    dims = api.make_dims(H, c.heads, c.head_dim, c.ffn)
    nts = api.adaln_modulation(dims, w["adaln_w"].cuda(), w["adaln_b"].cuda(),
                               w["adaln_table"].cuda(), 18 * H, L["segments"], L["seq_len"], sv, sa, out)
    assert nts == len(ts)
    got = f64(out[: nts * 18 * H]).reshape(nts * 3, 6 * H)
    np.testing.assert_allclose(got, ref, rtol=1e-4, atol=1e-6)


@pytest.mark.parametrize("rank", [6, 24, 32])
def test_adaln_modulation_ranks(cuda_ok, rank):
    # rank 24 and 32 take the coalesced prologue path (16-byte basis rows);
    # rank 6 (24-byte rows) takes the per-row kernel
    H = 256
    cfg = configs.DitConfig("r", 9, hidden=H, heads=2, head_dim=128, ffn=512, text_len=1, rank=rank)
    w = configs.block_weights(cfg, 0, keys=("adaln_w", "adaln_b", "adaln_table"))
    segs, _ = t2va_layout(20, 3, 16, 20, 20)
    n = segs[-1][1]
    sv, sa = sigma_pair(0.4)
    ts, _ = O.plan_timesteps(sv, sa, segs)
    ref = O.block_mods(f64(w["adaln_w"]), f64(w["adaln_b"]), f64(w["adaln_table"]), ts, H)
    out = torch.full((2 * 18 * H,), float("nan"), device="cuda")
    dims = api.make_dims(H, 2, 128, 512, rank=rank)
    nts = api.adaln_modulation(dims, w["adaln_w"].cuda(), w["adaln_b"].cuda(), w["adaln_table"].cuda(),
                               18 * H, segs, n, sv, sa, out)
    assert nts == 2
    np.testing.assert_allclose(f64(out[: nts * 18 * H]).reshape(6, 6 * H), ref, rtol=1e-4, atol=1e-6)


def t2va_layout(*a):
    L = O.layout_t2va(*a)
    return L["segments"], L["pos"]


def _qkv(n, heads, hd, seed, dtype=torch.bfloat16, qscale=1.0):
    I = heads * hd
    q = synth.normal((n, I), seed, qscale, dtype=dtype)
    k = synth.normal((n, I), seed + 1, 1.0, dtype=dtype)
    v = synth.normal((n, I), seed + 2, 1.0, dtype=dtype)
    return torch.cat([q, k, v], dim=1).contiguous()


@pytest.mark.parametrize("n,heads,hd", [(1, 2, 128), (127, 1, 128), (128, 2, 128), (129, 1, 128),
                                        (300, 3, 128), (1000, 2, 128), (300, 4, 64)])
def test_attention_bf16(cuda_ok, n, heads, hd):
    qkv = _qkv(n, heads, hd, 100 + n)
    out = torch.full((n, heads * hd), float("nan"), dtype=torch.bfloat16, device="cuda")
    api.attention(qkv.cuda(), 1, n, heads, hd, 1 / math.sqrt(hd), out)
    api.device_status()
    q, k, v = (f64(t).reshape(n, heads, hd) for t in qkv.split(heads * hd, dim=1))
    ref = O.attention(q, k, v, 1 / math.sqrt(hd)).reshape(n, -1)
    assert_close(out, ref, what=f"attention n={n}")


def test_attention_large_scores_exercise_rescale(cuda_ok):
    # scores with std ~6 make the running maximum grow by more than 2^8
    # between key tiles, so the O rescale path runs.
    n, heads, hd = 700, 2, 128
    qkv = _qkv(n, heads, hd, 7, qscale=6.0)
    out = torch.empty((n, heads * hd), dtype=torch.bfloat16, device="cuda")
    api.attention(qkv.cuda(), 1, n, heads, hd, 1 / math.sqrt(hd), out)
    api.device_status()
    q, k, v = (f64(t).reshape(n, heads, hd) for t in qkv.split(heads * hd, dim=1))
    ref = O.attention(q, k, v, 1 / math.sqrt(hd)).reshape(n, -1)
    assert_close(out, ref, what="attention large scores")


def test_attention_growing_maximum_every_tile(cuda_ok):
    # Scores that climb with the key index: along k's first dimension the
    # log2-domain score of an even query row rises by about 11 per key tile,
    # so its running maximum outgrows the reference on every tile, while odd
    # rows (a twentieth of the slope) rarely do.  Rows of both kinds share
    # each warp.
    n, heads, hd = 1000, 1, 128
    gen = torch.Generator().manual_seed(5)
    q = 0.05 * torch.randn((n, hd), generator=gen)
    k = 0.05 * torch.randn((n, hd), generator=gen)
    v = torch.randn((n, hd), generator=gen)
    q[:, 0] = torch.where(torch.arange(n) % 2 == 0, 1.0, 0.05)
    k[:, 0] = 0.06 * math.sqrt(hd) * torch.arange(n, dtype=torch.float32)
    qkv = torch.cat([q, k, v], dim=1).to(torch.bfloat16).contiguous()
    out = torch.empty((n, hd), dtype=torch.bfloat16, device="cuda")
    api.attention(qkv.cuda(), 1, n, heads, hd, 1 / math.sqrt(hd), out)
    api.device_status()
    q64, k64, v64 = (f64(t).reshape(n, heads, hd) for t in qkv.split(hd, dim=1))
    ref = O.attention(q64, k64, v64, 1 / math.sqrt(hd)).reshape(n, -1)
    assert_close(out, ref, what="attention growing maximum")


def test_attention_multi_sequence(cuda_ok):
    n_seq, seq, heads, hd = 3, 200, 2, 64
    qkv = _qkv(n_seq * seq, heads, hd, 11)
    out = torch.empty((n_seq * seq, heads * hd), dtype=torch.bfloat16, device="cuda")
    api.attention(qkv.cuda(), n_seq, seq, heads, hd, 0.125, out)
    api.device_status()
    for b in range(n_seq):
        part = qkv[b * seq:(b + 1) * seq]
        q, k, v = (f64(t).reshape(seq, heads, hd) for t in part.split(heads * hd, dim=1))
        ref = O.attention(q, k, v, 0.125).reshape(seq, -1)
        assert_close(out[b * seq:(b + 1) * seq], ref, what=f"sequence {b}")


@pytest.mark.parametrize("n_seq,seq,heads", [(1, 1, 1), (1, 64, 4), (1, 128, 1), (1, 129, 2), (1, 200, 2),
                                             (1, 300, 1), (3, 100, 2)])
def test_attention_fp32_tf32(cuda_ok, n_seq, seq, heads):
    # the fp32-storage path on the tensor cores (kind::tf32): one key tile,
    # ragged tiles, several tiles (online rescale) and several sequences
    hd = 64
    n = n_seq * seq
    qkv = _qkv(n, heads, hd, 21, dtype=torch.float32)
    out = torch.full((n, heads * hd), float("nan"), dtype=torch.float32, device="cuda")
    api.attention(qkv.cuda(), n_seq, seq, heads, hd, 1 / 8, out)
    assert api.status_sync() == 0
    for b in range(n_seq):
        part = qkv[b * seq:(b + 1) * seq]
        q, k, v = (f64(t).reshape(seq, heads, hd) for t in part.split(heads * hd, dim=1))
        ref = O.attention(q, k, v, 1 / 8).reshape(seq, -1)
        assert_close(out[b * seq:(b + 1) * seq], ref, TF32_MAXABS, TF32_COS, what=f"attention tf32 sequence {b}")


def test_attention_fp32_tf32_growing_scores(cuda_ok):
    # scores that grow along the keys: every key tile raises the row maximum,
    # so O is rescaled on every tile
    n, heads, hd = 384, 1, 64
    qkv = _qkv(n, heads, hd, 23, dtype=torch.float32)
    qkv[:, 0] = 1.0
    qkv[:, heads * hd] = 0.01 * math.sqrt(hd) * torch.arange(n, dtype=torch.float32)
    out = torch.empty((n, heads * hd), dtype=torch.float32, device="cuda")
    api.attention(qkv.cuda(), 1, n, heads, hd, 1 / 8, out)
    assert api.status_sync() == 0
    q, k, v = (f64(t).reshape(n, heads, hd) for t in qkv.split(heads * hd, dim=1))
    ref = O.attention(q, k, v, 1 / 8).reshape(n, -1)
    assert_close(out, ref, TF32_MAXABS, TF32_COS, what="attention tf32, growing scores")


def test_bounded_wait_returns_timeout_and_context_survives(cuda_ok):
    assert api.selftest_wait_timeout(1_000_000) == 7      # MMH3_ERR_TIMEOUT after ~1 ms
    assert api.device_status() == (0, 0)                  # status was cleared
    n, heads, hd = 130, 1, 128
    qkv = _qkv(n, heads, hd, 5)
    out = torch.empty((n, heads * hd), dtype=torch.bfloat16, device="cuda")
    api.attention(qkv.cuda(), 1, n, heads, hd, 1 / math.sqrt(hd), out)
    api.device_status()
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("n_seq,seq,heads,hd", [(1, 700, 5, 128), (1, 12288, 1, 128), (2, 8192, 1, 64),
                                                (1, 13248, 21, 128)])
def test_attention_split_tail(cuda_ok, n_seq, seq, heads, hd):
    # last-wave units split along the keys (partials + merge) against the
    # oracle and against the unsplit kernel: 700 keys are too few to split;
    # 12288 keys x 1 head (48 units) split in three; two sequences of 8192
    # (64 units, head_dim 64) in two; the block workload's 1092 units (56 in
    # the last wave) in two
    n = n_seq * seq
    qkv = _qkv(n, heads, hd, 300 + seq).cuda()
    scale = 1 / math.sqrt(hd)
    out = torch.full((n, heads * hd), float("nan"), dtype=torch.bfloat16, device="cuda")
    scratch = torch.empty(160 * 256 * (hd + 4) * 4, dtype=torch.uint8, device="cuda")
    c0 = api.launch_count()
    api.attention_ws(qkv, n_seq, seq, heads, hd, scale, out, scratch)
    # the whole units and the split tail are one grid; a split adds only the merge
    assert api.launch_count() - c0 == (1 if seq == 700 else 2)
    plain = torch.empty_like(out)
    api.attention(qkv, n_seq, seq, heads, hd, scale, plain)
    api.device_status()
    assert_close(out, plain, 4e-3, 0.99999, "split tail vs unsplit", rel=2.0 ** -8)
    rows = range(n) if n <= 1000 else range(0, n, 97)
    for b in range(n_seq):
        part = qkv[b * seq:(b + 1) * seq].cpu()
        q, k, v = (f64(t).reshape(seq, heads, hd) for t in part.split(heads * hd, dim=1))
        sel = [r - b * seq for r in rows if b * seq <= r < (b + 1) * seq]
        ref = O.attention(q, k, v, scale, q_rows=np.asarray(sel)).reshape(len(sel), -1)
        assert_close(out[b * seq:(b + 1) * seq][sel], ref, what=f"split tail sequence {b}")


@pytest.mark.parametrize("n_seq,seq,heads,hd", [(4, 2048, 21, 128), (32, 1024, 12, 64), (200, 100, 2, 64),
                                                (3, 700, 8, 128)])
def test_attention_persistent_matches_one_cta_per_item(cuda_ok, n_seq, seq, heads, hd):
    # a 256-byte scratch holds only the work counter: the launch is
    # persistent (148 CTAs, each walking several items through the work
    # ring; 100-key sequences give one-tile items) and nothing is split, so
    # every item computes exactly what the launch without scratch (one CTA
    # per item) computes: equal bit for bit, and sampled rows against the
    # oracle
    n = n_seq * seq
    qkv = _qkv(n, heads, hd, 500 + seq).cuda()
    scale = 1 / math.sqrt(hd)
    out = torch.full((n, heads * hd), float("nan"), dtype=torch.bfloat16, device="cuda")
    counter_only = torch.empty(256, dtype=torch.uint8, device="cuda")
    c0 = api.launch_count()
    api.attention_ws(qkv, n_seq, seq, heads, hd, scale, out, counter_only)
    assert api.launch_count() - c0 == 1
    plain = torch.empty_like(out)
    api.attention(qkv, n_seq, seq, heads, hd, scale, plain)
    assert api.status_sync() == 0
    assert torch.equal(out, plain)
    for b in (0, n_seq - 1):
        part = qkv[b * seq:(b + 1) * seq].cpu()
        q, k, v = (f64(t).reshape(seq, heads, hd) for t in part.split(heads * hd, dim=1))
        sel = np.arange(0, seq, 37)
        ref = O.attention(q, k, v, scale, q_rows=sel).reshape(len(sel), -1)
        assert_close(out[b * seq:(b + 1) * seq][sel.tolist()], ref, what=f"persistent, sequence {b}")


def test_attention_split_tail_with_rescales(cuda_ok):
    # 12288 keys x 1 head split in three with scores of std ~5: rows rescale
    # inside each piece, the pieces end with different reference maxima, and
    # the merge weighs them by 2^(m_p - max m); sampled rows against the
    # oracle, every row against the unsplit kernel
    n, heads, hd = 12288, 1, 128
    qkv = _qkv(n, heads, hd, 41, qscale=5.0).cuda()
    scale = 1 / math.sqrt(hd)
    out = torch.full((n, heads * hd), float("nan"), dtype=torch.bfloat16, device="cuda")
    scratch = torch.empty(160 * 256 * (hd + 4) * 4, dtype=torch.uint8, device="cuda")
    api.attention_ws(qkv, 1, n, heads, hd, scale, out, scratch)
    plain = torch.empty_like(out)
    api.attention(qkv, 1, n, heads, hd, scale, plain)
    api.device_status()
    # P is rounded to bf16 against each piece's own reference maximum, so the
    # two kernels differ by more than rounding order: the oracle's bf16 bar
    assert_close(out, plain, BF16_MAXABS, BF16_COS, "split tail with rescales vs unsplit")
    rows = np.arange(0, n, 89)
    q, k, v = (f64(t).reshape(n, heads, hd) for t in qkv.cpu().split(heads * hd, dim=1))
    ref = O.attention(q, k, v, scale, q_rows=rows).reshape(len(rows), -1)
    assert_close(out[rows.tolist()], ref, what="split tail with rescales")
