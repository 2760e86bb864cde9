"""Benchmark of the packed DiT block (MiniMax-H3 shape) on B200.

Workload (N = 1): one MiniMax-H3-shaped block, hidden 2688, 21 x 128 heads,
SwiGLU 10752, packed sequence of 13 248 tokens = text 256 + audio 2 x 256 +
video 8 x 30 x 52 (t2va layout, two flow clocks, sigma_v = 0.5), bf16 GEMM
operands, fp32 residual stream, seeded synthetic weights and inputs.  One
step = one mmh3_block_forward call: timestep plan, adaLN curve, segment-gather
RMSNorm + modulate, qkv GEMM + qk-norm + 3-axis rotation, attention, out GEMM
+ gated residual, RMSNorm + modulate, fc1 GEMM + SwiGLU, fc2 GEMM + gated
residual.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

With N > 1 (torchrun, one rank per GPU) every rank runs an independent
replica of the workload (the path has no exchange step); the reported time
is the maximum over ranks and the value is all ranks' tokens over it.
`--impl reference` times the CPU oracle on the host cores instead (one whole
block of the same workload per step).
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "packed DiT block tokens/s (bf16, 1 B200); attn/GEMM % tensor peak"
UNIT = "tokens/s"
N_TOKENS = 13248
PROFILE_PAUSE_S = 2.0  # idle time between the timed pass and the profile pass
WORKLOAD = ("MiniMax-H3 block: hidden 2688, 21x128 heads, SwiGLU 10752, packed seq 13248 = "
            "text 256 + audio 2x256 + video 8x30x52 (t2va, 2 timesteps, sigma_v 0.5)")


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", default="b200", choices=["b200", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--workload", default="block",
                   choices=["block", "stack", "image", "siglip", "tiny", "cp", "refine", "denoise"],
                   help="block (default) prints the benchmark line; the others print one JSON line "
                        "each for the remaining workloads (stack: 50 blocks + heads, image: 50 "
                        "blocks, siglip: one encoder layer x 32 images, tiny: fp32 block, cp: the "
                        "block over 2 and 4 sequence shards run one after another on one GPU, "
                        "refine: the token refiner, denoise: one whole denoise call at the stack "
                        "shape with embed and unpacking)")
    return p.parse_args()


# ------------------------------------------------------------------ peaks
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# --------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled every few
    milliseconds while the timed region runs: read-only NVML queries on a
    background thread (nvidia-smi as a fallback when NVML cannot be loaded).
    The GPU is found by its PCI bus id, so CUDA_VISIBLE_DEVICES remapping does
    not matter."""

    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40}

    def __init__(self, cuda_device: int, period_s: float = 0.005):
        self.dev = cuda_device
        self.period = period_s
        self.samples = []          # (sm_mhz, reasons bitmask)
        self.sm_max = None
        self.source = None
        self._stop = threading.Event()
        self._thread = None
        self._proc = None

    def _nvml_handle(self):
        import pynvml as N
        import torch
        N.nvmlInit()
        props = torch.cuda.get_device_properties(self.dev)
        try:
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            h = N.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            h = N.nvmlDeviceGetHandleByIndex(self.dev)
        return N, h

    def _run_nvml(self, N, h):
        get_reasons = getattr(N, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            N.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append((float(N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM)), int(get_reasons(h))))
            except Exception:
                pass
            time.sleep(self.period)

    def _run_smi(self):
        for line in self._proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            try:
                mhz, mx = float(parts[0]), float(parts[1])
            except (ValueError, IndexError):
                continue
            self.sm_max = mx
            bits = 0
            for (name, bit), v in zip(self.REASONS.items(), parts[2:6]):
                if v.lower().startswith("active"):
                    bits |= bit
            self.samples.append((mhz, bits))

    def __enter__(self):
        try:
            N, h = self._nvml_handle()
            self.sm_max = float(N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM))
            self.source = "nvml"
            self._thread = threading.Thread(target=self._run_nvml, args=(N, h), daemon=True)
        except Exception:
            try:
                self._proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.dev}",
                     "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.sw_power_cap,"
                     "clocks_event_reasons.hw_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                     "clocks_event_reasons.hw_thermal_slowdown",
                     "--format=csv,noheader,nounits", "-lms", "20"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.source = "nvidia-smi"
                self._thread = threading.Thread(target=self._run_smi, daemon=True)
            except Exception:
                self._thread = None
        if self._thread is not None:
            self._thread.start()
            t0 = time.time()
            while not self.samples and time.time() - t0 < 3.0:   # the first sample before the timed region
                time.sleep(0.002)
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except Exception:
                self._proc.kill()
        if self._thread is not None:
            self._thread.join(timeout=2)

    def summary(self):
        sm = [m for m, _ in self.samples]
        reasons = sorted({name for _, bits in self.samples for name, bit in self.REASONS.items() if bits & bit})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.sm_max,
                "reasons": reasons, "samples": len(sm), "source": self.source}


# ------------------------------------------------------ multi-rank timing
def max_over_ranks(ms: float, device, world: int) -> float:
    """The slowest rank's device time (every rank gets the same value)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tokens_per_rank: int, steps: int, ms_max: float) -> float:
    """Whole-job tokens/s: every rank runs `steps` replicas of the workload,
    the job takes as long as its slowest rank."""
    return world * tokens_per_rank * steps / (ms_max / 1e3)


# -------------------------------------------------- ncu traffic of a kernel
def measured_traffic(record: str):
    """DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per step of
    the dominant kernel from a JSON record under profiles/ that
    profile_summary.py wrote from an ncu capture, or None when the record is
    missing or any source file it lists has changed since (its sha256 no
    longer matches)."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", record)) as f:
            rec = json.load(f)
        for path, digest in rec["sources"].items():
            with open(os.path.join(ROOT, path), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest() != digest:
                    return None
        return int(rec["traffic_bytes_per_step"])
    except (OSError, KeyError, ValueError):
        return None


# ------------------------------------------------------- algorithmic work
def block_flops(n, H=2688, I=2688, F=10752):
    gemm = {"qkv gemm": 2.0 * n * H * 3 * I, "out gemm": 2.0 * n * I * H,
            "fc1 gemm": 2.0 * n * H * 2 * F, "fc2 gemm": 2.0 * n * F * H}
    gemm["attention"] = 4.0 * n * n * I
    return gemm


def hbm_bytes(n, H=2688, k=16, t_s=2, rank=24, blocks_per_prologue=1, act_bytes=2):
    """Algorithmic HBM bytes per launch of the memory-bound kernels:
    RMSNorm + modulate reads x (fp32) and writes xn (act dtype); the
    prologue reads each block's adaLN basis [T_s*18H, R] and bias and writes
    its modulation (fp32), and writes the rotation table ((cos, sin) fp32
    pairs from the positions)."""
    norm = n * H * 4 + n * H * act_bytes
    return {"norm1": norm, "norm2": norm,
            "prologue": blocks_per_prologue * t_s * 18 * H * (rank * 4 + 4 + 4) + n * 3 * 4 + n * 3 * k * 8}


def hbm_fractions(kernels, hb, peak_gbs):
    """Per memory-bound kernel: mean event time per launch, bytes, GB/s and
    the fraction of the HBM peak."""
    out = {}
    for name, nbytes in hb.items():
        kms, calls = kernels.get(name, (0.0, 0))
        if calls:
            t = kms / calls
            gbs = nbytes / (t / 1e3) / 1e9
            out[name] = {"ms_per_launch": round(t, 5), "launches": calls, "bytes_per_launch": nbytes,
                         "achieved_gbs": round(gbs, 1), "frac": round(gbs / peak_gbs, 4)}
    return out


def percentile(v, q):
    """Linear-interpolation percentile of a list (q in [0, 100])."""
    v = sorted(v)
    if not v:
        return None
    x = (len(v) - 1) * q / 100.0
    lo = int(math.floor(x))
    hi = min(lo + 1, len(v) - 1)
    return v[lo] + (v[hi] - v[lo]) * (x - lo)


def choose_peak(peaks, clocks, timed_s):
    """The bf16 peak the timed region ran against: the burst figure while the
    SM clock stayed at its maximum (a short run, not power-capped), the
    sustained (power-capped) figure otherwise.  Without clock samples the
    length of the timed region decides (under one second: burst)."""
    sm, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    if sm and mx:
        burst = sm >= 0.97 * mx
        why = f"median SM clock {sm:.0f} of max {mx:.0f} MHz under load"
    else:
        burst = timed_s < 1.0
        why = f"no clock samples; timed region {timed_s:.2f} s"
    kind = "burst" if burst else "sustained"
    return (peaks["bf16_tflops"] if burst else peaks["bf16_tflops_sustained"]), kind, why


# ------------------------------------------------------------- GPU arm
def build_workload(device):
    import numpy as np
    import torch

    from packed_multimodal_diffusion_b200 import api, configs
    c = configs.BLOCK
    segs, pos = api.layout_t2va(c.text_len, c.latent_t, c.lat_h, c.lat_w, c.audio_t)
    n = pos.shape[0]
    assert n == N_TOKENS
    dims = api.make_dims(c.hidden, c.heads, c.head_dim, c.ffn)
    # weights generated on the device from the same counter-based streams
    w = configs.block_weights(c, 0, device=device)
    params = api.BlockParams.from_host(dims, w, device=device)
    x0 = configs.hidden_states(c, device=device)
    pos_d = torch.as_tensor(pos.astype(np.float32), device=device)
    ws = torch.empty(api.workspace_size(dims, n), dtype=torch.uint8, device=device)
    sv = c.sigma_v
    sa = api.time_shift_sigma(sv, 12.0, 3.0)
    return dict(c=c, segs=segs, pos=pos, n=n, dims=dims, params=params, x0=x0, pos_d=pos_d,
                ws=ws, sv=sv, sa=sa)


def run_gpu(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    from packed_multimodal_diffusion_b200 import api

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = f"cuda:{local}"
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device(device))

    def barrier():
        if world > 1:
            dist.barrier()

    W = build_workload(device)
    x = W["x0"].clone()
    stream = torch.cuda.current_stream()

    def step():
        api.block_forward(W["dims"], W["params"], x, W["segs"], W["pos_d"], W["sv"], W["sa"], W["ws"])

    for _ in range(max(3, args.warmup)):
        step()
    api.device_status()

    # ---- device-timed region: one event before every step and one after
    # the last (the per-step distribution).  No per-kernel events here: an
    # event between two kernels orders the second after the first's
    # completion and undoes the programmatic launch overlap of the block's
    # kernels.
    barrier()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    launches0 = api.launch_count()
    with ClockSampler(torch.cuda.current_device()) as clk:
        ev[0].record(stream)
        for i in range(args.steps):
            step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
    launches = api.launch_count() - launches0
    barrier()
    ms = ev[0].elapsed_time(ev[-1])
    per_step = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    api.device_status()
    ms_max = max_over_ranks(ms, device, world)

    # ---- profile pass: the same steps again with the phase profiler's
    # per-kernel events (the phase and per-kernel times, and the dominant
    # kernel's time for the roofline).  The 1 kW power cap lowers the clock
    # after about ten steps; an idle pause and the same warm-up start this
    # pass from the power state the timed pass started from.
    time.sleep(PROFILE_PAUSE_S)
    for _ in range(max(3, args.warmup)):
        step()
    api.prof_reset()
    api.prof_enable(True)
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize()
    api.prof_enable(False)
    phases, nblocks = api.prof_collect()
    kernels = api.prof_collect_kernels()
    api.device_status()

    # ---- the same step replayed from a CUDA graph (one stream capture of
    # the block's launches), from the power state the timed pass started from
    time.sleep(PROFILE_PAUSE_S)
    for _ in range(max(3, args.warmup)):
        step()
    g_per, g_ms, g_kernels, g_clocks = time_graph(step, args.steps, max(3, args.warmup))
    api.device_status()
    g_ms_max = max_over_ranks(g_ms, device, world)

    # ---- end to end through the C ABI with host buffers (pinned), copies
    # inside the timed region: each step copies its input in and its result
    # out (mmh3_block_forward_host); three device slots let a step's
    # copy-out and a later step's copy-in overlap the blocks between them
    x_host = W["x0"].cpu().pin_memory()
    pos_host = torch.as_tensor(np.asarray(W["pos"], np.float32)).pin_memory()
    out_host = [torch.empty_like(x_host).pin_memory() for _ in range(api.HOST_SLOTS)]
    xd = [torch.empty_like(W["x0"]) for _ in range(api.HOST_SLOTS)]
    pd = [torch.empty_like(W["pos_d"]) for _ in range(api.HOST_SLOTS)]
    copy_in, copy_out = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)
    # at least 30 steps: the first copy-in and the last copy-out (about
    # 2.6 ms each at the block workload) are the pipeline's fill and drain
    e2e_steps = max(30, args.steps)
    e2e_count = [0]

    def e2e_step():
        k = e2e_count[0] % api.HOST_SLOTS
        e2e_count[0] += 1
        api.block_forward_host(W["dims"], W["params"], x_host, out_host[k], W["segs"], pos_host, W["sv"],
                               W["sa"], k, xd[k], pd[k], W["ws"], copy_in, copy_out)

    for _ in range(3):
        e2e_step()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    copy_in.wait_event(e0)
    copy_out.wait_event(e0)
    for _ in range(e2e_steps):
        e2e_step()
    stream.wait_stream(copy_out)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), device, world)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return

    n = W["n"]
    step_ms = ms_max / args.steps
    value = job_throughput(world, n, args.steps, ms_max)
    flops = block_flops(n)
    per_launch = {k: v / max(1, nblocks) for k, v in phases.items() if v > 0}
    dom = max(("attention", "qkv gemm", "out gemm", "fc1 gemm", "fc2 gemm"),
              key=lambda k: per_launch.get(k, 0.0))
    traffic = measured_traffic("attn2_block_13248.traffic.json") if dom == "attention" else None
    peaks = load_peaks()
    clocks = clk.summary()
    peak, peak_kind, peak_why = choose_peak(peaks, clocks, ms / 1e3)
    achieved = flops[dom] / (per_launch[dom] / 1e3) / 1e12
    total_flop = sum(flops.values())
    hbm_kernels = hbm_fractions(kernels, hbm_bytes(n), peaks["hbm_gbs"])
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_dict(world),
        "step_ms": {"median": statistics.median(per_step), "p10": percentile(per_step, 10),
                    "p90": percentile(per_step, 90), "mean": ms / args.steps},
        "tflops_per_s": total_flop / (step_ms / 1e3) / 1e12,
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"{peaks['source']} bf16 {peak_kind} (MEASURED_PEAKS.json)"
                                    if peaks["source"] == "measured" else
                                    f"fallback bf16 {peak_kind} (profiling recipe; MEASURED_PEAKS.json absent)",
                     "peak_kind": peak_kind, "peak_reason": peak_why,
                     "frac_burst": achieved / peaks["bf16_tflops"],
                     "frac_sustained": achieved / peaks["bf16_tflops_sustained"],
                     "traffic": traffic,
                     "traffic_unit": ("bytes per attention step (the attention launch, whole units and "
                                      "split tail in one grid, and the merge when the tail is split)"
                                      if dom == "attention"
                                      else "bytes/launch"),
                     "algorithmic_bytes": 2 * n * 3 * 2688 + 2 * n * 2688},
        "phases_ms_per_block": {k: round(v / max(1, nblocks), 4) for k, v in phases.items()},
        "phase_frac_of_peak": {k: round(flops[k] / (per_launch[k] / 1e3) / 1e12 / peak, 4)
                               for k in flops if k in per_launch},
        "hbm_kernels": {"peak_gbs": peaks["hbm_gbs"], "peak_source": peaks["source"], **hbm_kernels},
        "e2e": {"value": job_throughput(world, n, e2e_steps, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": int(W["x0"].numel() * 4 + W["pos_d"].numel() * 4),
                "d2h_bytes_per_step": int(W["x0"].numel() * 4)},
        "gpu_launches": launches,
        "clocks": clocks,
        "graph": {"value": job_throughput(world, n, args.steps, g_ms_max), "unit": UNIT,
                  **graph_entry(g_per, g_ms_max, g_kernels, g_clocks, args.steps)},
    }
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline()
    print(json.dumps(line), flush=True)


def config_dict(world: int) -> dict:
    return {"workload": WORKLOAD, "n_tokens": N_TOKENS, "hidden": 2688, "heads": 21, "head_dim": 128,
            "ffn": 10752, "timesteps": 2,
            "l2": "inputs larger than L2 (x 142 MB fp32, weights 231 MB bf16), no flush",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


# -------------------------------------------------------------- CPU oracle
class OracleBlock:
    """The oracle (fp64 numpy, as it stands) on the whole block workload,
    timed as one whole block cut into `parts` contiguous chunks of query
    rows: the first chunk's call also evaluates the adaLN modulation and k
    and v of every token (the oracle's k/v cache hands them to the later
    chunks), so the chunks together do exactly one block's work, and their
    times add up to one measured block.  Inputs are generated and widened
    before any timing."""

    def __init__(self):
        from oracle import mmh3_oracle as O
        from packed_multimodal_diffusion_b200 import configs
        self.O = O
        c = self.c = configs.BLOCK
        L = self.L = O.layout_t2va(c.text_len, c.latent_t, c.lat_h, c.lat_w, c.audio_t)
        self.n = L["seq_len"]
        w = configs.block_weights(c, 0)
        self.p = {k: v.double().numpy() for k, v in w.items()}
        self.x = configs.hidden_states(c).double().numpy()
        sa = O.time_shift_sigma(c.sigma_v, 12.0, 3.0)
        self.ts, slot = O.plan_timesteps(c.sigma_v, sa, L["segments"])
        self.rows = O.token_rows(L["segments"], slot, self.n)
        try:
            from threadpoolctl import threadpool_info
            self.cores = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
        except Exception:
            self.cores = os.cpu_count()

    def block_in_parts(self, parts: int) -> list:
        """Seconds of each of the `parts` chunks of one whole block."""
        import numpy as np
        O, c, p = self.O, self.c, self.p
        bounds = np.linspace(0, self.n, max(1, min(parts, self.n)) + 1).astype(int)
        cache, mods, times = {}, None, []
        for a, b in zip(bounds[:-1], bounds[1:]):
            t0 = time.perf_counter()
            if mods is None:
                mods = O.block_mods(p["adaln_w"], p["adaln_b"], p["adaln_table"], self.ts, c.hidden)
            O.block_forward(p, self.x, mods, self.rows, self.L["pos"], c.dims(),
                            sample_rows=np.arange(a, b), kv_cache=cache)
            times.append(time.perf_counter() - t0)
        return times

    def describe(self, times) -> str:
        return (f"one whole block of the block workload ({self.n} tokens: adaLN modulation, k/v of every "
                f"token and all {self.n} query rows through the block, fp64 numpy) in {len(times)} "
                f"timed chunk(s) of query rows, {sum(times):.1f} s in total")


def cpu_baseline():
    o = OracleBlock()
    times = o.block_in_parts(1)
    return {"value": o.n / sum(times), "unit": UNIT, "cores": o.cores, "kind": "oracle",
            "sample": o.describe(times)}


def run_reference(args):
    """The reference arm: the CPU oracle.  The `steps` timed steps together
    compute one whole block (each a contiguous chunk of the query rows, the
    first also the modulation and k/v of every token), so the value is the
    block's tokens over the measured time of one block.  The oracle keeps no
    state between blocks, so there is nothing to warm up and no warm-up block
    runs (the line records the requested count).  Only rank 0 runs it."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    o = OracleBlock()
    times = o.block_in_parts(args.steps)
    total = sum(times)
    value = o.n / total
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": len(times),
            "warmup": 0, "warmup_requested": args.warmup, "ms_per_step": 1e3 * total / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference", "config": config_dict(1),
            "step_ms": {"median": 1e3 * statistics.median(times), "p10": 1e3 * percentile(times, 10),
                        "p90": 1e3 * percentile(times, 90), "mean": 1e3 * total / len(times)},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": o.cores, "kind": "oracle",
                             "sample": o.describe(times)},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------- other workloads
def _time(fn, steps, warmup):
    """Mean ms per call of fn over `steps` calls after `warmup`, CUDA events
    on the current stream, with the clocks sampled meanwhile."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
    _time.clocks = clk.summary()
    return e0.elapsed_time(e1) / steps


def time_graph(fn, steps, warmup):
    """`fn` captured once into a CUDA graph (stream capture; the library's
    launches, programmatic edges included, become the graph's nodes), then
    `warmup` untimed replays and `steps` timed ones, with a CUDA event on the
    current stream before every replay and after the last.  Returns the
    per-replay ms, the total ms, the library kernels one replay launches and
    the clocks sampled while timing."""
    import torch

    from packed_multimodal_diffusion_b200 import api
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    k0 = api.launch_count()
    with torch.cuda.graph(g):
        fn()
    kernels = api.launch_count() - k0
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    with ClockSampler(torch.cuda.current_device()) as clk:
        ev[0].record()
        for i in range(steps):
            g.replay()
            ev[i + 1].record()
        torch.cuda.synchronize()
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
    total = ev[0].elapsed_time(ev[-1])
    g.reset()
    return per, total, kernels, clk.summary()


def graph_entry(per, total, kernels, clocks, steps) -> dict:
    return {"ms_per_step": total / steps,
            "step_ms": {"median": statistics.median(per), "p10": percentile(per, 10),
                        "p90": percentile(per, 90), "mean": total / steps},
            "kernels_per_step": kernels, "clocks": clocks}


def run_workload(args):
    """One JSON line for the stack, image, SigLIP or tiny workload (device-timed
    with CUDA events, weights generated on the device from the seeded streams,
    per-phase profile from a second pass over the same steps)."""
    import numpy as np
    import torch

    from packed_multimodal_diffusion_b200 import api, configs
    torch.cuda.set_device(0)
    dev = "cuda"
    steps, warmup = max(1, args.steps), max(1, args.warmup)
    peaks = load_peaks()
    line = {"workload": args.workload, "data": "synthetic", "steps": steps, "warmup": warmup}
    if args.workload == "siglip":
        c = configs.SIGLIP
        d = api.vit_dims(c.hidden, c.heads, c.head_dim, c.mlp, c.ln_eps)
        params = api.VitParams.from_host(d, configs.vit_weights(c, device=dev), device=dev)
        x = configs.vit_inputs(c, device=dev)
        ws = torch.empty(api.vit_workspace_size(d, c.batch, c.seq), dtype=torch.uint8, device=dev)
        ms = _time(lambda: api.vit_layer_forward(d, params, x, c.batch, c.seq, ws), steps, warmup)
        clocks = _time.clocks
        api.device_status()
        graph = graph_entry(*time_graph(lambda: api.vit_layer_forward(d, params, x, c.batch, c.seq, ws),
                                        steps, warmup), steps)
        api.device_status()
        # the phase profiler's pass over the same number of layers
        api.prof_reset()
        api.prof_enable(True)
        for _ in range(steps):
            api.vit_layer_forward(d, params, x, c.batch, c.seq, ws)
        torch.cuda.synchronize()
        api.prof_enable(False)
        phases, nlayers = api.prof_collect()
        kernels = api.prof_collect_kernels()
        api.device_status()
        rows = c.batch * c.seq
        # LayerNorm reads x (fp32) and writes its bf16 output once
        ln_bytes = rows * c.hidden * 4 + rows * c.hidden * 2
        hbm_ln = hbm_fractions(kernels, {"norm1": ln_bytes, "norm2": ln_bytes}, peaks["hbm_gbs"])
        H, Fm = c.hidden, c.mlp
        vflops = {"qkv gemm": 2.0 * rows * H * 3 * H, "attention": 4.0 * c.batch * c.seq ** 2 * H,
                  "out gemm": 2.0 * rows * H * H, "fc1 gemm": 2.0 * rows * H * Fm, "fc2 gemm": 2.0 * rows * Fm * H}
        per_layer = {k: v / max(1, nlayers) for k, v in phases.items() if v > 0}
        peak, _, _ = choose_peak(peaks, clocks, ms * steps / 1e3)
        flop = sum(vflops.values())
        line.update(metric="SigLIP encoder layer time (bf16, 1 B200)", value=ms, unit="ms/layer",
                    higher_is_better=False, dtype="bf16", tokens_per_s=rows / (ms / 1e3),
                    tflops_per_s=flop / (ms / 1e3) / 1e12,
                    config={"workload": "SigLIP layer: 32 images x 1024 tokens, hidden 768, 12x64 heads, "
                                        "MLP 3072 tanh-GELU, LayerNorm pre-norm"},
                    context="the pages quote 61.9 ms/layer for batch 1 on an unnamed CPU",
                    phases_ms_per_layer={k: round(v, 4) for k, v in per_layer.items()},
                    phase_frac_of_peak={k: round(vflops[k] / (per_layer[k] / 1e3) / 1e12 / peak, 4)
                                        for k in vflops if k in per_layer},
                    peak_tflops=peak,
                    hbm_kernels={"peak_gbs": peaks["hbm_gbs"], "peak_source": peaks["source"],
                                 **{("ln1" if k == "norm1" else "ln2"): v for k, v in hbm_ln.items()}},
                    clocks=clocks, graph={"value": graph["ms_per_step"], "unit": "ms/layer", **graph})
        print(json.dumps(line), flush=True)
        return
    c = {"stack": configs.STACK, "image": configs.IMAGE, "tiny": configs.TINY}[args.workload]
    if c.image_mode:
        segs, pos = api.layout_image(c.text_len, c.ref_lat_h, c.ref_lat_w, c.lat_h, c.lat_w)
    else:
        segs, pos = api.layout_t2va(c.text_len, c.latent_t, c.lat_h, c.lat_w, c.audio_t)
    n = pos.shape[0]
    dims = api.make_dims(c.hidden, c.heads, c.head_dim, c.ffn, act_dtype=c.act_dtype)
    blocks = [api.BlockParams.from_host(dims, configs.block_weights(c, b, device=dev), device=dev)
              for b in range(c.n_blocks)]
    x0 = configs.hidden_states(c, device=dev)
    x = x0.clone()
    pd = torch.as_tensor(pos.astype(np.float32), device=dev)
    ws = torch.empty(api.workspace_size(dims, n), dtype=torch.uint8, device=dev)
    sv = c.sigma_v
    sa = api.time_shift_sigma(max(sv, 1e-6), 12.0, 3.0)
    heads = None
    ov = oa = None
    if c.heads_out or c.image_mode:
        hc = c if c.heads_out else configs.DitConfig(c.name, c.cfg_seed, hidden=c.hidden, heads=c.heads,
                                                       head_dim=c.head_dim, ffn=c.ffn, text_len=c.text_len,
                                                       heads_out=128)
        heads = api.HeadParams.from_host(configs.head_weights(hc, device=dev), device=dev)
        vseg = [sg for sg in segs if sg[2] == 0][-1]
        aseg = [sg for sg in segs if sg[2] == 2]
        ov = torch.empty((vseg[1] - vseg[0], 128), device=dev)
        oa = torch.empty((aseg[-1][1] - aseg[-1][0], 128), device=dev) if aseg else None

    def step():
        x.copy_(x0)
        api.stack_forward(dims, blocks, heads, x, segs, pd, sv, sa, ov, oa, ws)

    # timed without per-kernel events (they would undo the programmatic
    # launch overlap), then the same steps again with the phase profiler
    ms = _time(step, steps, warmup)
    clocks = _time.clocks
    api.prof_reset()
    api.prof_enable(True)
    for _ in range(steps):
        step()
    torch.cuda.synchronize()
    api.prof_enable(False)
    phases, nblocks = api.prof_collect()
    kernels = api.prof_collect_kernels()
    api.device_status()
    graph = graph_entry(*time_graph(step, steps, warmup), steps)
    api.device_status()
    flops = block_flops(n, c.hidden, c.heads * c.head_dim, c.ffn)
    per_block = {k: v / max(1, nblocks) for k, v in phases.items() if v > 0}
    peak, peak_kind, _ = choose_peak(peaks, clocks, ms * steps / 1e3)
    line.update(clocks=clocks, peak_tflops=peak, peak_kind=peak_kind)
    line.update(metric=f"{args.workload} forward time (1 B200)", value=ms, unit="ms/forward",
                higher_is_better=False, dtype="fp32/tf32" if c.act_dtype == torch.float32 else "bf16",
                n_tokens=n, n_blocks=c.n_blocks, heads=bool(heads),
                tokens_per_s_per_block=n * c.n_blocks / (ms / 1e3),
                tflops_per_s=c.n_blocks * sum(flops.values()) / (ms / 1e3) / 1e12,
                phases_ms_per_block={k: round(v, 4) for k, v in per_block.items()},
                phase_frac_of_peak={k: round(flops[k] / (per_block[k] / 1e3) / 1e12 / peak, 4)
                                    for k in flops if k in per_block},
                hbm_kernels={"peak_gbs": peaks["hbm_gbs"], "peak_source": peaks["source"],
                             **hbm_fractions(kernels, hbm_bytes(
                                 n, c.hidden, c.rope_k, len(api.plan_timesteps(segs, n, sv, sa)[0]), c.rank,
                                 blocks_per_prologue=min(c.n_blocks, 64),
                                 act_bytes=4 if c.act_dtype == torch.float32 else 2), peaks["hbm_gbs"])},
                config={"workload": f"{c.name}: n {n}, hidden {c.hidden}, {c.heads}x{c.head_dim} heads, "
                                    f"SwiGLU {c.ffn}, {c.n_blocks} blocks" + (", output heads" if heads else "")},
                graph={"value": graph["ms_per_step"], "unit": "ms/forward", **graph})
    print(json.dumps(line), flush=True)


def run_next(args):
    """JSON lines for the rows around the block: the block over sequence
    shards (context parallel; the shards run one after another on one GPU,
    so the time is the compute of all shards, without any exchange), the
    token refiner, and one whole denoise call (embed, 50 blocks, heads,
    unpacking) at the stack shape."""
    import numpy as np
    import torch

    from packed_multimodal_diffusion_b200 import api, configs, shard
    torch.cuda.set_device(0)
    dev = "cuda"
    steps, warmup = max(1, args.steps), max(1, args.warmup)
    line = {"workload": args.workload, "data": "synthetic", "steps": steps, "warmup": warmup,
            "higher_is_better": False, "dtype": "bf16"}
    if args.workload == "cp":
        c = configs.BLOCK
        segs, pos = api.layout_t2va(c.text_len, c.latent_t, c.lat_h, c.lat_w, c.audio_t)
        n = pos.shape[0]
        dims = api.make_dims(c.hidden, c.heads, c.head_dim, c.ffn)
        params = api.BlockParams.from_host(dims, configs.block_weights(c, 0, device=dev), device=dev)
        x0 = configs.hidden_states(c, device=dev)
        pd = torch.as_tensor(pos.astype(np.float32), device=dev)
        sv = c.sigma_v
        sa = api.time_shift_sigma(max(sv, 1e-6), 12.0, 3.0)
        inner = c.heads * c.head_dim
        ws1 = torch.empty(api.workspace_size(dims, n), dtype=torch.uint8, device=dev)
        x1 = x0.clone()
        one = _time(lambda: api.block_forward(dims, params, x1, segs, pd, sv, sa, ws1), steps, warmup)
        del ws1
        worlds = {}
        for world in (2, 4):
            m, parts = shard.shard_rows(n, world)
            kv_all = torch.empty((world * m, 2 * inner), dtype=torch.bfloat16, device=dev)
            xs = [x0[r0:r0 + rows].clone() for r0, rows in parts]
            wss = [torch.empty(api.workspace_size(dims, max(rows, 1)), dtype=torch.uint8, device=dev)
                   for _, rows in parts]
            ssegs = [shard.shard_segments(segs, r0, rows) for r0, rows in parts]
            pss = [pd[r0:r0 + rows].clone() for r0, rows in parts]

            def run():
                for r, (r0, rows) in enumerate(parts):
                    api.block_cp_begin(dims, params, xs[r], ssegs[r], pss[r], sv, sa, kv_all[r * m:r * m + rows],
                                       wss[r])
                for r, (r0, rows) in enumerate(parts):
                    api.block_cp_end(dims, params, xs[r], ssegs[r], sv, sa, kv_all, n, wss[r])

            ms = _time(run, steps, warmup)
            api.device_status()
            worlds[f"shards_{world}"] = {"ms_all_shards": ms, "ms_per_shard": ms / world,
                                         "rows_per_shard": m, "kv_exchange_bytes_per_rank": 2 * n * 2 * inner}
            del wss, kv_all
        line.update(metric="block over sequence shards, compute only (bf16, 1 B200)", value=one,
                    unit="ms/block (one GPU, whole sequence)", shards=worlds,
                    config={"workload": f"block: n {n}, hidden 2688, 21x128 heads, SwiGLU 10752; shards "
                                        "emulated one after another on one GPU, K|V gathered in place"},
                    clocks=_time.clocks)
    elif args.workload == "refine":
        c = configs.BLOCK
        text_dim, n_blocks, n = 4096, 2, c.text_len
        dims = api.make_dims(c.hidden, c.heads, c.head_dim, c.ffn)
        sd = lambda j: configs.synth.tensor_seed(7, 800 + j)  # noqa: E731
        states = configs.synth.normal((n, text_dim), sd(0), 1.0, dtype=torch.bfloat16, device=dev)
        cond_w = configs.synth.normal((c.hidden, text_dim), sd(1), text_dim ** -0.5, dtype=torch.bfloat16,
                                      device=dev)
        cond_b = configs.synth.normal((c.hidden,), sd(2), 0.1, device=dev)
        norm = configs.synth.normal((c.hidden,), sd(3), 0.1, 1.0, device=dev)
        blocks = [api.BlockParams.from_host(dims, configs.block_weights(c, 10 + b, device=dev), device=dev)
                  for b in range(n_blocks)]
        out = torch.empty((n, c.hidden), dtype=torch.float32, device=dev)
        ws = torch.empty(api.refine_workspace_size(dims, n), dtype=torch.uint8, device=dev)
        ms = _time(lambda: api.refine_text(dims, states, cond_w, cond_b, blocks, norm, 1e-6, out, ws), steps,
                   warmup)
        api.device_status()
        line.update(metric="token refiner time (bf16, 1 B200)", value=ms, unit="ms/call",
                    config={"workload": f"token refiner: {n} text tokens of width {text_dim} (assumed), "
                                        f"projection to hidden 2688, {n_blocks} unmodulated unrotated blocks "
                                        "(21x128 heads, SwiGLU 10752), final RMSNorm"},
                    clocks=_time.clocks)
    else:  # denoise
        c = configs.STACK
        segs, pos = api.layout_t2va(c.text_len, c.latent_t, c.lat_h, c.lat_w, c.audio_t)
        n = pos.shape[0]
        H, Cv, Ca = c.hidden, c.heads_out // 4, c.heads_out
        dims = api.make_dims(c.hidden, c.heads, c.head_dim, c.ffn)
        sd = lambda j: configs.synth.tensor_seed(8, 900 + j)  # noqa: E731
        text = configs.synth.normal((c.text_len, H), sd(0), 1.0, device=dev)
        video = configs.synth.normal((Cv, c.latent_t, c.lat_h, c.lat_w), sd(1), 1.0, device=dev)
        audio = configs.synth.normal((Ca, 2, c.audio_t), sd(2), 1.0, device=dev)
        ew = (configs.synth.normal((H, 4 * Cv), sd(3), (4 * Cv) ** -0.5, dtype=torch.bfloat16, device=dev),
              configs.synth.normal((H,), sd(4), 0.1, device=dev),
              configs.synth.normal((H, Ca), sd(5), Ca ** -0.5, dtype=torch.bfloat16, device=dev),
              configs.synth.normal((H,), sd(6), 0.1, device=dev))
        blocks = [api.BlockParams.from_host(dims, configs.block_weights(c, b, device=dev), device=dev)
                  for b in range(c.n_blocks)]
        heads = api.HeadParams.from_host(configs.head_weights(c, device=dev), device=dev)
        pd = torch.as_tensor(pos.astype(np.float32), device=dev)
        x = torch.empty((n, H), device=dev)
        vo = torch.empty_like(video)
        ao = torch.empty_like(audio)
        ws = torch.empty(api.forward_workspace_size(dims, n, text, video, audio), dtype=torch.uint8, device=dev)
        sv = c.sigma_v
        sa = api.time_shift_sigma(max(sv, 1e-6), 12.0, 3.0)
        ms = _time(lambda: api.forward(dims, segs, n, pd, sv, sa, text, video, audio, ew, blocks, heads, x, vo,
                                       ao, ws), steps, warmup)
        clocks = _time.clocks
        ews = torch.empty(api.embed_workspace_size(dims, text, video, audio), dtype=torch.uint8, device=dev)
        ms_embed = _time(lambda: api.embed(dims, segs, n, text, video, audio, *ew, x, ews), steps, warmup)
        vseg = [sg for sg in segs if sg[2] == 0][-1]
        aseg = [sg for sg in segs if sg[2] == 2]
        vrows = torch.empty((vseg[1] - vseg[0], 4 * Cv), device=dev)
        arows = torch.empty((aseg[-1][1] - aseg[0][0], Ca), device=dev)

        def unpack():
            api.unpatchify_video(vrows, Cv, c.latent_t, c.lat_h, c.lat_w, vo)
            api.unpack_audio(arows, Ca, c.audio_t, ao)

        ms_unpack = _time(unpack, steps, warmup)
        api.device_status()
        line.update(metric="denoise call time (bf16, 1 B200)", value=ms, unit="ms/call",
                    embed_ms=ms_embed, unpack_ms=ms_unpack,
                    config={"workload": f"one denoise evaluation at the stack shape: embed (text {c.text_len} x "
                                        f"{H}, video latents {Cv}x{c.latent_t}x{c.lat_h}x{c.lat_w} patchified "
                                        f"2x2, audio {Ca}x2x{c.audio_t}), 50 blocks (n {n}), both heads "
                                        "(128 each), unpatchify and audio unpacking"},
                    clocks=clocks)
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.workload in ("cp", "refine", "denoise"):
        run_next(args)
    elif args.workload != "block":
        run_workload(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
