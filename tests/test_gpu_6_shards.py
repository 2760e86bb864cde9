"""GPU parity of the block over sequence shards (mmh3_block_cp_begin /
mmh3_block_cp_end): the ranks of a context-parallel run are emulated one
after another on one GPU, the K|V exchange is the gathered buffer the begin
calls fill in place, and the shards' outputs are compared with the oracle's
block over the whole sequence and with the single-GPU block."""

import pytest

from gpu_common import (BF16_COS, BF16_MAXABS, BF16_STORE_REL, api, assert_close, configs, f64, np,
                        oracle_block, sigma_pair, small_block_weights, small_dims, t2va, torch)
from packed_multimodal_diffusion_b200 import shard

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world,layout", [(2, (20, 3, 16, 20, 20)), (3, (20, 3, 16, 20, 20)),
                                          (4, (5, 1, 4, 4, 3)), (2, (130, 2, 16, 16, 64))])
def test_sharded_block_matches_whole_sequence(cuda_ok, world, layout):
    dims_o, dims_c = small_dims()
    segs, pos = t2va(*layout)
    n = int(pos.shape[0])
    w = small_block_weights(41, 256, 2, 128, 512)
    x = configs.synth.normal((n, 256), 91, 1.0)
    sv, sa = sigma_pair(0.5)
    params = api.BlockParams.from_host(dims_c, w)
    inner = 2 * 128
    m, shards = shard.shard_rows(n, world)
    pos_d = torch.as_tensor(np.asarray(pos, np.float32)).cuda()
    kv_all = torch.full((world * m, 2 * inner), float("nan"), dtype=torch.bfloat16, device="cuda")
    xs, wss = [], []
    for r, (row0, rows) in enumerate(shards):
        xs.append(x[row0:row0 + rows].cuda().contiguous().clone())
        wss.append(torch.empty(api.workspace_size(dims_c, max(rows, 1)), dtype=torch.uint8, device="cuda"))
        if rows:
            api.block_cp_begin(dims_c, params, xs[r], shard.shard_segments(segs, row0, rows),
                               pos_d[row0:row0 + rows].clone(), sv, sa, kv_all[r * m:r * m + rows], wss[r])
    for r, (row0, rows) in enumerate(shards):
        if rows:
            api.block_cp_end(dims_c, params, xs[r], shard.shard_segments(segs, row0, rows), sv, sa,
                             kv_all, n, wss[r])
    api.device_status()
    out = torch.cat([t for t in xs if t.shape[0]], 0)
    ref, _, _ = oracle_block(w, x, segs, pos, sv, sa, dims_o)
    assert_close(out, ref, BF16_MAXABS, BF16_COS, "sharded x_out")
    assert_close(out.cpu().double() - x.double(), ref - f64(x), BF16_MAXABS, BF16_COS, "sharded delta")
    # against the whole-sequence block on one GPU: the same arithmetic per row
    # except for how the GEMM rows are tiled
    xw = x.cuda().clone()
    ws = torch.empty(api.workspace_size(dims_c, n), dtype=torch.uint8, device="cuda")
    api.block_forward(dims_c, params, xw, segs, pos_d, sv, sa, ws)
    assert_close(out, xw, 2e-3, 0.999999, "sharded vs single-GPU block", rel=2.0 ** -8)


@pytest.mark.parametrize("world", [2, 4])
def test_sharded_block_workload_full_size(cuda_ok, world):
    # the 13 248-token block over 2 and 4 shards against the single-GPU block
    # (the same arithmetic per row, up to how the GEMM rows are tiled) and,
    # on rows spanning text, audio, video and every shard, against the oracle
    c = configs.BLOCK
    segs, pos = t2va(c.text_len, c.latent_t, c.lat_h, c.lat_w, c.audio_t)
    n = int(pos.shape[0])
    w = configs.block_weights(c, 0)
    x = configs.hidden_states(c)
    sv, sa = sigma_pair(c.sigma_v)
    dims_c = api.make_dims(c.hidden, c.heads, c.head_dim, c.ffn)
    params = api.BlockParams.from_host(dims_c, w)
    inner = c.heads * c.head_dim
    m, shards = shard.shard_rows(n, world)
    pos_d = torch.as_tensor(np.asarray(pos, np.float32)).cuda()
    kv_all = torch.full((world * m, 2 * inner), float("nan"), dtype=torch.bfloat16, device="cuda")
    xs, wss = [], []
    for r, (row0, rows) in enumerate(shards):
        xs.append(x[row0:row0 + rows].cuda().contiguous().clone())
        wss.append(torch.empty(api.workspace_size(dims_c, rows), dtype=torch.uint8, device="cuda"))
        api.block_cp_begin(dims_c, params, xs[r], shard.shard_segments(segs, row0, rows),
                           pos_d[row0:row0 + rows].clone(), sv, sa, kv_all[r * m:r * m + rows], wss[r])
    for r, (row0, rows) in enumerate(shards):
        api.block_cp_end(dims_c, params, xs[r], shard.shard_segments(segs, row0, rows), sv, sa, kv_all, n,
                         wss[r])
    assert api.status_sync() == 0
    out = torch.cat(xs, 0)
    del wss
    xw = x.cuda().clone()
    ws = torch.empty(api.workspace_size(dims_c, n), dtype=torch.uint8, device="cuda")
    api.block_forward(dims_c, params, xw, segs, pos_d, sv, sa, ws)
    assert_close(out, xw, 2e-3, 0.999999, "sharded vs single-GPU block", rel=2.0 ** -8)
    sample = [0, 255, 256, 767, 768, m - 1, m, n // 2, n - 1]
    ref, _, _ = oracle_block(w, x, segs, pos, sv, sa, c.dims(), sample_rows=sample)
    assert_close(out[sample], ref, what="sharded x_out rows")
    assert_close(out[sample].cpu().double() - x[sample].double(), ref - f64(x[sample]), what="sharded delta rows")
