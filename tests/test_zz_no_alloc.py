"""The no-allocation block entry point (mmh3_block_forward_noalloc) gives the
same result as mmh3_block_forward with a caller workspace.

That entry point exists for callers that cannot allocate device memory --
for example a plugin whose host owns all device memory through its own pool,
or a runtime that must keep cudaMalloc (a device-synchronising call) off its
hot path.  It keeps the block's intermediates in one fixed library-owned
device array instead of a caller workspace.  This file is collected last so
that a run stopping at the first failure has already run every other test.
"""

import ctypes as C

import pytest
import torch

from gpu_common import (BF16_COS, BF16_MAXABS, api, assert_close, configs, np, sigma_pair,
                        small_block_weights, t2va)
from packed_multimodal_diffusion_b200 import _lib

pytestmark = pytest.mark.gpu


def _poison(dims, seed):
    """A no-alloc call on other data and a larger size, so that the shared
    scratch holds stale values everywhere the next call could read."""
    segs, pos = t2va(30, 4, 16, 24, 40)          # 30 + 80 + 384 = 494 tokens
    n = int(pos.shape[0])
    params = api.BlockParams.from_host(dims, small_block_weights(seed, 256, 2, 128, 512))
    x = configs.synth.normal((n, 256), seed + 1, 3.0).cuda()
    pd = torch.as_tensor(np.asarray(pos, np.float32)).cuda()
    api.block_forward_noalloc(dims, params, x, segs, pd, *sigma_pair(0.9))
    api.device_status()


def test_noalloc_block_matches_workspace_block_twice(cuda_ok):
    dims = api.make_dims(256, 2, 128, 512)
    segs, pos = t2va(20, 3, 16, 20, 20)          # 300 tokens, ragged last tile
    n = int(pos.shape[0])
    w = small_block_weights(91, 256, 2, 128, 512)
    params = api.BlockParams.from_host(dims, w)
    x = configs.synth.normal((n, 256), 92, 1.0).cuda()
    pd = torch.as_tensor(np.asarray(pos, np.float32)).cuda()
    sv, sa = sigma_pair(0.5)

    ws = torch.empty(api.workspace_size(dims, n), dtype=torch.uint8, device="cuda")
    ref = x.clone()
    api.block_forward(dims, params, ref, segs, pd, sv, sa, ws)
    api.device_status()

    for call in range(2):                           # two calls in a row share the scratch
        # another workload leaves different values in the scratch first, so a
        # read of a region before this call writes it would show
        _poison(dims, 400 + call)
        got = x.clone()
        api.block_forward_noalloc(dims, params, got, segs, pd, sv, sa)
        api.device_status()
        assert_close(got, ref, BF16_MAXABS, BF16_COS, what=f"no-alloc call {call}")
        assert_close(got - x, ref - x, BF16_MAXABS, BF16_COS, what=f"no-alloc call {call} delta")
        # the same kernels on the same inputs: identical to the last bit
        assert torch.equal(got, ref), f"no-alloc call {call} differs from the workspace block"


def test_noalloc_rejects_sizes_beyond_the_fixed_scratch(cuda_ok):
    dims = api.make_dims(2688, 21, 128, 10752)
    x = torch.zeros((600, 2688), device="cuda")
    w = {k: torch.zeros(1, device="cuda") for k in ("norm1", "norm2", "wqkv", "wout", "q_norm",
                                                    "k_norm", "wfc1_tiled", "wfc2", "adaln_w",
                                                    "adaln_b", "adaln_table")}
    with pytest.raises(_lib.Mmh3Error) as e:
        api.block_forward_noalloc(dims, api.BlockParams(w), x, [(0, 600, 1, 0)], None, 0.5, 0.2)
    assert e.value.code == 4
    assert "at most 556 tokens fit" in str(e.value)
