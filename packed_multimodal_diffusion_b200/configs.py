"""Workload shapes and the synthetic-input recipe.

Five workloads, named by what they are:

* ``tiny``   -- one block, hidden 256, 4 x 64 heads, SwiGLU 1024, packed
                sequence 64 = text 16 + audio 8 frames x 2 channels + video
                2 x 4 x 4 (latent 8 x 8), t_v = 0.7.
* ``block``  -- one MiniMax-H3-shaped block, hidden 2688, 21 x 128 heads,
                SwiGLU 10752, sequence 13 248 = text 256 + audio 256 x 2 +
                video 8 x 30 x 52 (latent 60 x 104).
* ``stack``  -- 50 such blocks plus the video and audio output heads
                (128 channels each), sequence 26 496 = text 512 + audio
                512 x 2 + video 16 x 30 x 52.
* ``image``  -- image mode, 50 blocks, one clock, sequence 8 448 = text 256
                + reference 64 x 64 patches + target 64 x 64 patches.
* ``siglip`` -- one unmodulated pre-norm ViT layer, 32 images x 1024 tokens,
                hidden 768, 12 x 64 heads, MLP 3072 with tanh-GELU.

Recipe: projections, adaLN basis and biases N(0, 0.02); norm gains
1 + N(0, 0.02); the timestep-curve table N(0, 1); hidden states N(0, 1).
Each tensor has its own SplitMix64 stream, seed ``cfg_seed*1000 + index``.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch

from . import synth


@dataclass(frozen=True)
class DitConfig:
    name: str
    cfg_seed: int
    hidden: int
    heads: int
    head_dim: int
    ffn: int
    text_len: int
    # t2va: latent_t frames of lat_h x lat_w latents (2x2 patches) + audio_t
    # audio frames per channel.  image mode: ref_lat / lat are the reference
    # and target latent grids.
    latent_t: int = 0
    lat_h: int = 0
    lat_w: int = 0
    audio_t: int = 0
    image_mode: bool = False
    ref_lat_h: int = 0
    ref_lat_w: int = 0
    n_blocks: int = 1
    sigma_v: float = 0.5
    heads_out: int = 0          # output-head channels (0: no heads)
    act_dtype: torch.dtype = torch.bfloat16
    rope_theta: float = 10000.0
    eps: float = 1e-5
    qk_eps: float = 1e-5
    rank: int = 24
    grid: int = 1025

    @property
    def inner(self) -> int:
        return self.heads * self.head_dim

    @property
    def rope_k(self) -> int:
        """Frequencies per position axis: the rotated span is 3/4 of a head
        (48 pairs of a 128-dim head), so k = head_dim / 8."""
        return self.head_dim // 8

    @property
    def seq_len(self) -> int:
        if self.image_mode:
            return (self.text_len + (self.ref_lat_h // 2) * (self.ref_lat_w // 2)
                    + (self.lat_h // 2) * (self.lat_w // 2))
        return (self.text_len + 2 * self.audio_t
                + self.latent_t * (self.lat_h // 2) * (self.lat_w // 2))

    @property
    def n_slots(self) -> int:
        """adaLN timestep slots the basis carries: two clocks."""
        return 2

    def dims(self) -> dict:
        return dict(hidden=self.hidden, heads=self.heads, head_dim=self.head_dim,
                    ffn=self.ffn, eps=self.eps, qk_eps=self.qk_eps,
                    rope_k=self.rope_k, rope_theta=self.rope_theta)


@dataclass(frozen=True)
class VitConfig:
    name: str
    cfg_seed: int
    batch: int
    seq: int
    hidden: int
    heads: int
    head_dim: int
    mlp: int
    ln_eps: float = 1e-6

    def dims(self) -> dict:
        return dict(hidden=self.hidden, heads=self.heads, head_dim=self.head_dim,
                    mlp=self.mlp, ln_eps=self.ln_eps)


TINY = DitConfig("tiny", 0, hidden=256, heads=4, head_dim=64, ffn=1024,
                 text_len=16, latent_t=2, lat_h=8, lat_w=8, audio_t=8,
                 sigma_v=0.3, act_dtype=torch.float32)
BLOCK = DitConfig("block", 1, hidden=2688, heads=21, head_dim=128, ffn=10752,
                  text_len=256, latent_t=8, lat_h=60, lat_w=104, audio_t=256)
STACK = DitConfig("stack", 2, hidden=2688, heads=21, head_dim=128, ffn=10752,
                  text_len=512, latent_t=16, lat_h=60, lat_w=104, audio_t=512,
                  n_blocks=50, heads_out=128)
IMAGE = DitConfig("image", 3, hidden=2688, heads=21, head_dim=128, ffn=10752,
                  text_len=256, image_mode=True, ref_lat_h=128, ref_lat_w=128,
                  lat_h=128, lat_w=128, n_blocks=50)
SIGLIP = VitConfig("siglip", 4, batch=32, seq=1024, hidden=768, heads=12,
                   head_dim=64, mlp=3072)

CONFIGS = {c.name: c for c in (TINY, BLOCK, STACK, IMAGE, SIGLIP)}

# tensor indices inside a config's seed space
_BLOCK_STRIDE = 16
_HEADS_BASE = 900
_X_INDEX = 990
_VIT_BASE = 800


def block_weights(cfg: DitConfig, b: int, device="cpu", wdtype=None, keys=None) -> dict:
    """Synthetic weights of block ``b`` (natural layouts: qkv rows [q|k|v],
    fc1 rows [gate|up]).  Projections in ``wdtype`` (default: the config's
    activation dtype), everything else fp32.  ``keys`` limits the output to
    those tensors (each has its own stream, so a subset is identical to the
    same entries of the full set)."""
    wdtype = cfg.act_dtype if wdtype is None else wdtype
    H, I, F, R = cfg.hidden, cfg.inner, cfg.ffn, cfg.rank
    base = b * _BLOCK_STRIDE
    s = lambda j: synth.tensor_seed(cfg.cfg_seed, base + j)  # noqa: E731
    n = synth.normal
    make = {
        "norm1": lambda: n((H,), s(0), 0.02, 1.0, device=device),
        "norm2": lambda: n((H,), s(1), 0.02, 1.0, device=device),
        "wqkv": lambda: n((3 * I, H), s(2), 0.02, dtype=wdtype, device=device),
        "wout": lambda: n((H, I), s(3), 0.02, dtype=wdtype, device=device),
        "q_norm": lambda: n((cfg.head_dim,), s(4), 0.02, 1.0, device=device),
        "k_norm": lambda: n((cfg.head_dim,), s(5), 0.02, 1.0, device=device),
        "wfc1": lambda: n((2 * F, H), s(6), 0.02, dtype=wdtype, device=device),
        "wfc2": lambda: n((H, F), s(7), 0.02, dtype=wdtype, device=device),
        "adaln_w": lambda: n((cfg.n_slots * 3 * 6 * H, R), s(8), 0.02, device=device),
        "adaln_b": lambda: n((cfg.n_slots * 3 * 6 * H,), s(9), 0.02, device=device),
        "adaln_table": lambda: n((cfg.grid, R), s(10), 1.0, device=device),
    }
    return {k: f() for k, f in make.items() if keys is None or k in keys}


def head_weights(cfg: DitConfig, device="cpu", wdtype=None) -> dict:
    """Synthetic final-layer weights: final RMSNorm gain, the final adaLN
    curve (one modality, chunks shift/scale) and the two output linears."""
    wdtype = cfg.act_dtype if wdtype is None else wdtype
    H, R, C = cfg.hidden, cfg.rank, cfg.heads_out
    s = lambda j: synth.tensor_seed(cfg.cfg_seed, _HEADS_BASE + j)  # noqa: E731
    n = synth.normal
    return {
        "final_norm": n((H,), s(0), 0.02, 1.0, device=device),
        "adaln_w": n((cfg.n_slots * 2 * H, R), s(1), 0.02, device=device),
        "adaln_b": n((cfg.n_slots * 2 * H,), s(2), 0.02, device=device),
        "adaln_table": n((cfg.grid, R), s(3), 1.0, device=device),
        "w_video": n((C, H), s(4), 0.02, dtype=wdtype, device=device),
        "b_video": n((C,), s(5), 0.02, device=device),
        "w_audio": n((C, H), s(6), 0.02, dtype=wdtype, device=device),
        "b_audio": n((C,), s(7), 0.02, device=device),
    }


def hidden_states(cfg: DitConfig, n: int | None = None, device="cpu") -> torch.Tensor:
    """Packed hidden states [n, H], N(0, 1), fp32."""
    n = cfg.seq_len if n is None else n
    return synth.normal((n, cfg.hidden), synth.tensor_seed(cfg.cfg_seed, _X_INDEX),
                        1.0, device=device)


def vit_weights(cfg: VitConfig, device="cpu", wdtype=torch.bfloat16) -> dict:
    """Synthetic SigLIP-layer weights (q, k, v, o, fc1, fc2 with biases;
    LayerNorm gains 1 + N(0, 0.02) and biases N(0, 0.02))."""
    H, M = cfg.hidden, cfg.mlp
    s = lambda j: synth.tensor_seed(cfg.cfg_seed, _VIT_BASE + j)  # noqa: E731
    n = synth.normal
    return {
        "ln1_g": n((H,), s(0), 0.02, 1.0, device=device),
        "ln1_b": n((H,), s(1), 0.02, device=device),
        "wq": n((H, H), s(2), 0.02, dtype=wdtype, device=device),
        "wk": n((H, H), s(3), 0.02, dtype=wdtype, device=device),
        "wv": n((H, H), s(4), 0.02, dtype=wdtype, device=device),
        "bq": n((H,), s(5), 0.02, device=device),
        "bk": n((H,), s(6), 0.02, device=device),
        "bv": n((H,), s(7), 0.02, device=device),
        "wo": n((H, H), s(8), 0.02, dtype=wdtype, device=device),
        "bo": n((H,), s(9), 0.02, device=device),
        "ln2_g": n((H,), s(10), 0.02, 1.0, device=device),
        "ln2_b": n((H,), s(11), 0.02, device=device),
        "w1": n((M, H), s(12), 0.02, dtype=wdtype, device=device),
        "b1": n((M,), s(13), 0.02, device=device),
        "w2": n((H, M), s(14), 0.02, dtype=wdtype, device=device),
        "b2": n((H,), s(15), 0.02, device=device),
    }


def vit_inputs(cfg: VitConfig, batch: int | None = None, device="cpu") -> torch.Tensor:
    """Patch embeddings [batch*seq, H], N(0, 1), fp32."""
    b = cfg.batch if batch is None else batch
    return synth.normal((b * cfg.seq, cfg.hidden),
                        synth.tensor_seed(cfg.cfg_seed, _X_INDEX), 1.0, device=device)
