"""Host logic of bench.py on CPU.  Two gloo ranks (the path has no exchange
step, so ranks are independent replicas) agree on the slowest rank's time,
and the whole-job value counts every rank's tokens over it.  The roofline's
ncu traffic is read from a JSON record only while the kernel sources still
match the capture; the peak follows the clock the run saw."""

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
    # the bench's roofline traffic comes from a JSON record that
    # profile_summary.py writes from an ncu CSV, and only while every source
    # file the record lists still has the sha256 recorded with the capture
    import json
    sys.path.insert(0, ROOT)
    import bench
    import profile_summary
    src = tmp_path / "kern.cuh"
    src.write_bytes(b"// kernel v1\n")
    (tmp_path / "profiles").mkdir()
    csv_text = "==PROF== header line\n" + "\n".join([
        '"ID","Kernel Name","Metric Name","Metric Unit","Metric Value"',
        '"0","attn2_tc_kernel(args)","dram__bytes_read.sum","Mbyte","200.5"',
        '"0","attn2_tc_kernel(args)","dram__bytes_write.sum","Kbyte","1,500"',
        '"0","attn2_tc_kernel(args)","gpu__time_duration.sum","msecond","1.5"',
        '"1","attn_merge_kernel(args)","dram__bytes_read.sum","byte","1000"',
        '"1","attn_merge_kernel(args)","dram__bytes_write.sum","byte","24"',
        '"1","attn_merge_kernel(args)","gpu__time_duration.sum","us","8"',
        '"2","gemm_tc_kernel(args)","dram__bytes_read.sum","byte","77"',
    ]) + "\n"
    (tmp_path / "cap.csv").write_text(csv_text)
    monkeypatch.chdir(tmp_path)
    out = tmp_path / "profiles" / "rec.json"
    monkeypatch.setattr(sys, "argv", ["profile_summary.py", "--csv", "cap.csv", "--kernels",
                                      "attn2_tc_kernel|attn_merge_kernel", "--per-step", "2",
                                      "--sources", "kern.cuh", "--workload", "w", "--command", "ncu ...",
                                      "--out", str(out)])
    profile_summary.main()
    rec = json.loads(out.read_text())
    assert rec["traffic_bytes_per_step"] == 200_500_000 + 1_500_000 + 1024
    assert rec["groups"][0]["kernels"] == ["attn2_tc_kernel", "attn_merge_kernel"]
    assert abs(rec["groups"][0]["duration_s"] - 1.508e-3) < 1e-12
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("rec.json") == rec["traffic_bytes_per_step"]
    src.write_bytes(b"// kernel v2\n")
    assert bench.measured_traffic("rec.json") is None
    assert bench.measured_traffic("missing.json") is None


def test_peak_choice_and_percentiles():
    sys.path.insert(0, ROOT)
    import bench
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    assert bench.choose_peak(peaks, {"sm_mhz": 1965, "sm_max_mhz": 1965}, 5.0)[:2] == (1600.0, "burst")
    assert bench.choose_peak(peaks, {"sm_mhz": 1500, "sm_max_mhz": 1965}, 0.1)[:2] == (1400.0, "sustained")
    assert bench.choose_peak(peaks, {"sm_mhz": None, "sm_max_mhz": None}, 0.1)[1] == "burst"
    assert bench.choose_peak(peaks, {"sm_mhz": None, "sm_max_mhz": None}, 3.0)[1] == "sustained"
    v = [4.0, 1.0, 3.0, 2.0, 5.0]
    assert bench.percentile(v, 50) == 3.0 and bench.percentile(v, 10) == pytest.approx(1.4)
    assert bench.percentile(v, 90) == pytest.approx(4.6)
    hb = bench.hbm_bytes(13248)
    assert hb["norm1"] == 13248 * 2688 * 6
    assert hb["prologue"] == 2 * 18 * 2688 * 104 + 13248 * 12 + 13248 * 48 * 8
    assert bench.hbm_bytes(64, blocks_per_prologue=50)["prologue"] == 50 * 2 * 18 * 2688 * 104 + 64 * 12 + 64 * 384
