"""CPU test of the sequence-shard host logic over real ranks (gloo,
world sizes 2 and 3): the shard rows, the shard segment tables, and the K|V
all-gather in block_forward_sharded, with the two compute halves replaced
by CPU stand-ins that write and check global row numbers."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from packed_multimodal_diffusion_b200 import shard

SEGS = [(0, 7, 1, 0), (7, 19, 2, 1), (19, 53, 0, 0)]
N = 53


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, failures):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        m, shards = shard.shard_rows(N, world)
        row0, rows = shards[rank]
        seen = {}

        def begin(dims, params, x, segs, pos, sv, sa, kv_out, ws, modulated):
            seen["segs"] = segs
            # K|V rows carry their global row number
            kv_out.copy_(torch.arange(row0, row0 + rows, dtype=torch.float32)[:, None].expand(rows, 2))

        def end(dims, params, x, segs, sv, sa, kv_all, n_kv, ws, modulated):
            assert n_kv == N
            assert torch.equal(kv_all[:N, 0], torch.arange(N, dtype=torch.float32))
            x += kv_all[row0:row0 + rows, :1]

        x = torch.zeros(rows, 1)
        kv_local = torch.full((m, 2), -1.0)
        kv_all = torch.empty(world * m, 2)
        shard.block_forward_sharded(None, None, x, SEGS, row0, N, None, 0.5, 0.2, kv_local, kv_all,
                                    None, begin=begin, end=end)
        assert torch.equal(x[:, 0], torch.arange(row0, row0 + rows, dtype=torch.float32))
        # the shard tables, moved back by their first rows, tile the whole table
        out = [None] * world
        dist.all_gather_object(out, (row0, seen.get("segs", [])))
        if rank == 0:
            rebuilt = []
            for r0, segs in out:
                for (a, b, tag, clock) in segs:
                    if rebuilt and rebuilt[-1][1] == a + r0 and rebuilt[-1][2:] == (tag, clock):
                        rebuilt[-1] = (rebuilt[-1][0], b + r0, tag, clock)
                    else:
                        rebuilt.append((a + r0, b + r0, tag, clock))
            assert rebuilt == SEGS, rebuilt
    except Exception as e:  # reported to the parent
        failures.put(f"rank {rank}: {e!r}")
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_block_host_logic_over_gloo_ranks(world):
    ctx = mp.get_context("spawn")
    failures = ctx.Queue()
    mp.start_processes(_rank_main, args=(world, _free_port(), failures), nprocs=world, join=True,
                       start_method="spawn")
    assert failures.empty()


def test_shard_rows_and_segments():
    m, shards = shard.shard_rows(10, 4)
    assert m == 3 and shards == [(0, 3), (3, 3), (6, 3), (9, 1)]
    m, shards = shard.shard_rows(9, 4)
    assert shards[-1] == (9, 0)
    assert shard.shard_segments(SEGS, 5, 10) == [(0, 2, 1, 0), (2, 10, 2, 1)]
    assert shard.shard_segments(SEGS, 40, 20) == [(0, 13, 0, 0)]
