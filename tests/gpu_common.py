"""Shared helpers of the GPU parity tests: seeded inputs, oracle calls and
the comparison bars.

Bars (floating point):
  * bf16 path, block outputs and block deltas (x_out - x_in): max-abs <= 2e-2
    and cosine >= 0.9995.
  * bf16-stored intermediates (xn1, q, k, v after qk-norm + rotation, attn,
    xn2, act): cosine >= 0.9995 and, element-wise,
    |gpu - ref| <= 2e-2 + 2^-7 |ref| -- rounding a value to bf16 alone moves
    it by up to 2^-8 |ref|, which exceeds 2e-2 for |ref| > 5.
  * fp32 modulation vectors: |gpu - oracle| <= 1e-4 |oracle| + 1e-6.
  * fp32-storage path (tcgen05 kind::tf32 GEMMs and attention):
    max-abs <= 5e-3 and cosine >= 0.99995, intermediates + 2^-10 |ref| --
    tf32 rounding (2^-11 relative per operand) is 16x finer than bf16's 2^-7,
    so the bf16 bar tightened by about that factor.
Integer work (rows, positions): exact.
"""

from __future__ import annotations

import math

import numpy as np
import torch

from oracle import mmh3_oracle as O
from packed_multimodal_diffusion_b200 import api, configs, synth

BF16_MAXABS, BF16_COS = 2e-2, 0.9995
TF32_MAXABS, TF32_COS = 5e-3, 0.99995


def f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().numpy().astype(np.float64)
    return np.asarray(t, dtype=np.float64)


def cosine(a, b) -> float:
    a, b = f64(a).ravel(), f64(b).ravel()
    na, nb = np.linalg.norm(a), np.linalg.norm(b)
    if na == 0 and nb == 0:
        return 1.0
    return float(a @ b / (na * nb))


def assert_close(gpu, ref, maxabs=BF16_MAXABS, cos=BF16_COS, what="", rel=0.0):
    """max |gpu - ref| <= maxabs (+ rel * |ref| element-wise) and cosine >= cos.

    rel > 0 is used for intermediates the GPU stores in a low-precision type:
    rounding a value v to bf16 alone moves it by up to |v| * 2^-8, so such a
    tensor gets the element-wise bound maxabs + 2^-7 |ref| (storage rounding
    plus the same again for the rounding of its bf16 inputs)."""
    g, r = f64(gpu), f64(ref)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite GPU values"
    excess = np.abs(g - r) - rel * np.abs(r)
    err = float(np.max(excess)) if g.size else 0.0
    c = cosine(g, r)
    assert err <= maxabs and c >= cos, \
        f"{what}: max-abs {err:.3e} beyond {rel:g}|ref| (bar {maxabs}), cosine {c:.6f} (bar {cos})"
    return err, c


#: element-wise relative allowance for bf16-stored intermediates
BF16_STORE_REL = 2.0 ** -7
#: the same for tf32-rounded GEMM inputs with fp32 storage
TF32_STORE_REL = 2.0 ** -10


def small_dims(hidden=256, heads=2, head_dim=128, ffn=512, act=torch.bfloat16):
    return dict(hidden=hidden, heads=heads, head_dim=head_dim, ffn=ffn, eps=1e-5, qk_eps=1e-5,
                rope_k=head_dim // 8, rope_theta=10000.0), api.make_dims(hidden, heads, head_dim,
                                                                         ffn, act_dtype=act)


def small_block_weights(seed, hidden, heads, head_dim, ffn, wdtype=torch.bfloat16):
    cfg = configs.DitConfig("small", seed, hidden=hidden, heads=heads, head_dim=head_dim, ffn=ffn,
                            text_len=1, act_dtype=wdtype)
    return configs.block_weights(cfg, 0, wdtype=wdtype)


def oracle_params(w: dict) -> dict:
    return {k: f64(v) for k, v in w.items()}


def oracle_block(w, x, segs, pos, sigma_v, sigma_a, dims, sample_rows=None, keep=None,
                 modulated=True):
    n = x.shape[0]
    ts, slot = O.plan_timesteps(sigma_v, sigma_a, segs)
    rows = O.token_rows(segs, slot, n)
    mods = O.block_mods(f64(w["adaln_w"]), f64(w["adaln_b"]), f64(w["adaln_table"]), ts,
                        dims["hidden"]) if modulated else None
    return O.block_forward(oracle_params(w), f64(x), mods, rows, None if pos is None else f64(pos),
                           dims, sample_rows=sample_rows, keep=keep), mods, rows


def t2va(text_len, latent_t, lat_h, lat_w, audio_t):
    L = O.layout_t2va(text_len, latent_t, lat_h, lat_w, audio_t)
    return L["segments"], L["pos"]


def sigma_pair(sigma_v):
    return sigma_v, O.time_shift_sigma(max(sigma_v, 1e-6), 12.0, 3.0)


def run_block(dims_c, w, x, segs, pos, sigma_v, sigma_a, modulated=True):
    """GPU block on copies of the inputs; returns (x_out, workspace regions)."""
    params = api.BlockParams.from_host(dims_c, w)
    xd = x.to("cuda").contiguous().clone()
    pd = None if pos is None else torch.as_tensor(np.asarray(pos, dtype=np.float32)).cuda()
    ws = torch.empty(api.workspace_size(dims_c, x.shape[0]), dtype=torch.uint8, device="cuda")
    api.block_forward(dims_c, params, xd, segs, pd, sigma_v, sigma_a, ws, modulated=modulated)
    api.device_status()
    return xd, api.workspace_regions(dims_c, x.shape[0], ws)


def heads_split(qkv, heads, head_dim):
    n = qkv.shape[0]
    I = heads * head_dim
    q = qkv[:, :I].reshape(n, heads, head_dim)
    k = qkv[:, I:2 * I].reshape(n, heads, head_dim)
    v = qkv[:, 2 * I:].reshape(n, heads, head_dim)
    return q, k, v


__all__ = ["O", "api", "configs", "synth", "math", "np", "torch"]
