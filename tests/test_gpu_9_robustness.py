"""Failure detection on the GPU without a fault: the check mode and the host
fault-injection sites that fire mid-block.

* MMH3_CHECK mode on (mmh3_set_check): the segment-row checks, the TMA
  coordinate checks and the workspace canaries run on valid inputs -- a
  small bf16 block (CTA-pair GEMMs), the fp32 tiny block (single-CTA tf32
  GEMMs), a stack with both heads and attention with a split last wave --
  record nothing, and every output equals the unchecked run bit for bit.
* MMH3_FAULT=tensormap / launch make the first GEMM of a block fail on the
  host after the prologue and the first RMSNorm were enqueued: the call
  returns MMH3_ERR_CUDA with the site's message, x is unchanged (only the
  GEMM epilogues write x), the device status is clean and the next call
  without the fault equals a reference call.
"""

import pytest

from gpu_common import (O, api, configs, np, sigma_pair, small_block_weights, small_dims, synth, t2va, torch)
from packed_multimodal_diffusion_b200 import _lib

pytestmark = pytest.mark.gpu


def _block_run(dims_c, w, x, segs, pos, sv, sa):
    params = api.BlockParams.from_host(dims_c, w)
    xd = x.cuda().clone()
    pd = torch.as_tensor(np.asarray(pos, np.float32)).cuda()
    ws = torch.empty(api.workspace_size(dims_c, x.shape[0]), dtype=torch.uint8, device="cuda")
    api.block_forward(dims_c, params, xd, segs, pd, sv, sa, ws)
    assert api.status_sync() == 0
    return xd.cpu()


@pytest.fixture
def check_mode():
    api.set_check(1)
    yield
    api.set_check(-1)
    api.status_sync()


def test_check_mode_block_fp32_block_and_stack_bit_identical(cuda_ok):
    dims_o, dims_c = small_dims()
    segs, pos = t2va(20, 3, 16, 20, 20)
    n = int(pos.shape[0])
    w = small_block_weights(111, 256, 2, 128, 512)
    x = configs.synth.normal((n, 256), 112, 1.0)
    sv, sa = sigma_pair(0.5)
    ref = _block_run(dims_c, w, x, segs, pos, sv, sa)
    c = configs.TINY
    L = O.layout_t2va(c.text_len, c.latent_t, c.lat_h, c.lat_w, c.audio_t)
    wt = configs.block_weights(c, 0)
    xt = configs.hidden_states(c)
    dims_t = api.make_dims(c.hidden, c.heads, c.head_dim, c.ffn, act_dtype=torch.float32)
    svt, sat = sigma_pair(c.sigma_v)
    ref_t = _block_run(dims_t, wt, xt, L["segments"], L["pos"], svt, sat)
    api.set_check(1)
    try:
        got = _block_run(dims_c, w, x, segs, pos, sv, sa)
        got_t = _block_run(dims_t, wt, xt, L["segments"], L["pos"], svt, sat)
        # a stack with heads, checked
        from test_gpu_3_stack_vit import _run_stack, _small_heads
        blocks = [small_block_weights(113 + i, 256, 2, 128, 512) for i in range(2)]
        heads = _small_heads(115, 256)
        xs_c, ov_c, oa_c = _run_stack(dims_c, blocks, heads, x, segs, pos, sv, sa)
        assert api.status_sync() == 0
    finally:
        api.set_check(-1)
    assert torch.equal(got, ref)
    assert torch.equal(got_t, ref_t)
    xs, ov, oa = _run_stack(dims_c, blocks, heads, x, segs, pos, sv, sa)
    assert torch.equal(xs_c, xs) and torch.equal(ov_c, ov) and torch.equal(oa_c, oa)


def test_check_mode_split_attention_bit_identical(cuda_ok):
    n, heads, hd = 12288, 1, 128          # 48 units: the last wave splits in three
    I = heads * hd
    qkv = torch.cat([synth.normal((n, I), 121 + i, 1.0, dtype=torch.bfloat16) for i in range(3)], dim=1).cuda()
    scratch = torch.empty(64 << 20, dtype=torch.uint8, device="cuda")
    out0 = torch.empty((n, I), dtype=torch.bfloat16, device="cuda")
    api.attention_ws(qkv, 1, n, heads, hd, hd ** -0.5, out0, scratch)
    assert api.status_sync() == 0
    api.set_check(1)
    try:
        out1 = torch.empty_like(out0)
        api.attention_ws(qkv, 1, n, heads, hd, hd ** -0.5, out1, scratch)
        assert api.status_sync() == 0
    finally:
        api.set_check(-1)
    assert torch.equal(out0, out1)


@pytest.mark.parametrize("site", ["tensormap", "launch"])
def test_mid_block_fault_injection_leaves_x_and_the_context_intact(cuda_ok, monkeypatch, site):
    dims_o, dims_c = small_dims()
    segs, pos = t2va(20, 3, 16, 20, 20)
    n = int(pos.shape[0])
    w = small_block_weights(131, 256, 2, 128, 512)
    x = configs.synth.normal((n, 256), 132, 1.0)
    sv, sa = sigma_pair(0.5)
    ref = _block_run(dims_c, w, x, segs, pos, sv, sa)
    params = api.BlockParams.from_host(dims_c, w)
    xd = x.cuda().clone()
    pd = torch.as_tensor(np.asarray(pos, np.float32)).cuda()
    ws = torch.empty(api.workspace_size(dims_c, n), dtype=torch.uint8, device="cuda")
    monkeypatch.setenv("MMH3_FAULT", site)
    with pytest.raises(_lib.Mmh3Error) as e:
        api.block_forward(dims_c, params, xd, segs, pd, sv, sa, ws)
    assert e.value.code == 6 and f"injected fault at {site}" in str(e.value)
    monkeypatch.delenv("MMH3_FAULT")
    assert api.status_sync() == 0
    assert torch.equal(xd.cpu(), x), "a block that failed before its first GEMM must leave x unchanged"
    api.block_forward(dims_c, params, xd, segs, pd, sv, sa, ws)
    assert api.status_sync() == 0
    assert torch.equal(xd.cpu(), ref)
