"""Host logic of bench.py on CPU.  Two gloo ranks (the path has no exchange
step, so ranks are independent replicas) agree on the slowest rank's time,
and the whole-job value counts every rank's tokens over it.  The roofline's
ncu traffic is read from a profile summary only while the kernel source
still matches the capture."""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [12.5, 40.0][rank]
        ms = bench.max_over_ranks(local_ms, "cpu", world)
        val = bench.job_throughput(world, 13248, 100, ms)
        out[rank] = (ms, val)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_count_all_tokens():
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(2, port, out), nprocs=2, start_method="spawn", join=True)
    assert out[0][0] == out[1][0] == 40.0
    assert out[0][1] == pytest.approx(2 * 13248 * 100 / 0.040)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.0, "cpu", 1) == 3.0
    assert bench.job_throughput(1, 10, 5, 1000.0) == 50.0


def test_measured_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    # the bench's roofline traffic comes from a profiles/ summary only while
    # the kernel source still has the sha256 recorded with the capture
    import hashlib
    sys.path.insert(0, ROOT)
    import bench
    src = tmp_path / "kern.cuh"
    src.write_bytes(b"// kernel v1\n")
    (tmp_path / "profiles").mkdir()
    digest = hashlib.sha256(src.read_bytes()).hexdigest()
    (tmp_path / "profiles" / "p.md").write_text(
        f"summary\n\ntraffic_bytes_per_step: 123456 source_sha256: {digest}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("p.md", "kern.cuh") == 123456
    src.write_bytes(b"// kernel v2\n")
    assert bench.measured_traffic("p.md", "kern.cuh") is None
    assert bench.measured_traffic("missing.md", "kern.cuh") is None

