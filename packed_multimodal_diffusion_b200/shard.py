"""Host side of the block over sequence shards (context parallelism).

The packed sequence of n rows is cut into contiguous shards of
m = ceil(n / world) rows, one per rank; the last shard may be shorter or
empty.  A block then runs as

    mmh3_block_cp_begin  (this rank's rows: norm1, qkv GEMM; K|V rows out)
    all-gather of the K|V rows over the ranks' process group
    mmh3_block_cp_end    (this rank's queries against all keys; the rest)

so the only exchange is the K|V all-gather, 2 * n * inner * 2 bytes per
block.  Rows of the gathered buffer beyond n are padding that the attention
kernel never reads.  This module holds only the row bookkeeping and the
collective call: every arithmetic step runs in libmmh3.so.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import api


def shard_rows(n: int, world: int) -> tuple[int, list[tuple[int, int]]]:
    """(m, [(first row, rows) per rank]) for n rows over `world` ranks."""
    if n < 1 or world < 1:
        raise ValueError("n and world must be positive")
    m = -(-n // world)
    return m, [(r * m, max(0, min(n, (r + 1) * m) - r * m)) for r in range(world)]


def shard_segments(segs, row0: int, rows: int) -> list[tuple]:
    """The segments a shard [row0, row0 + rows) intersects, with rows counted
    from the shard's first row (tags and clocks unchanged)."""
    out = []
    for (a, b, tag, clock) in segs:
        lo, hi = max(a, row0), min(b, row0 + rows)
        if lo < hi:
            out.append((lo - row0, hi - row0, tag, clock))
    return out


def block_forward_sharded(dims, params, x_loc: torch.Tensor, segs, row0: int, n: int,
                          pos_loc: torch.Tensor | None, sigma_v: float, sigma_a: float,
                          kv_local: torch.Tensor, kv_all: torch.Tensor, workspace: torch.Tensor,
                          group=None, modulated: bool = True,
                          begin=api.block_cp_begin, end=api.block_cp_end) -> None:
    """One block on this rank's shard, in place on x_loc [rows, H].

    segs: the whole sequence's segments; pos_loc: the shard's positions in a
    buffer of their own ([rows, 3] fp32, 16-byte aligned, so not a row slice
    of the whole sequence's positions); kv_local [m, 2*inner] and kv_all
    [world * m, 2*inner] bf16 buffers; workspace sized for m rows.  Every
    rank calls this (an empty shard still takes part in the all-gather)."""
    rows = x_loc.shape[0]
    segs_loc = shard_segments(segs, row0, rows)
    if rows > 0:
        begin(dims, params, x_loc, segs_loc, pos_loc, sigma_v, sigma_a, kv_local[:rows], workspace,
              modulated)
    dist.all_gather_into_tensor(kv_all, kv_local, group=group)
    if rows > 0:
        end(dims, params, x_loc, segs_loc, sigma_v, sigma_a, kv_all, n, workspace, modulated)
