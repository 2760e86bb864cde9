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
`--impl reference` times the CPU oracle on the host cores instead (a bounded
sample of the same workload per step).
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
WORKLOAD = ("MiniMax-H3 block: hidden 2688, 21x128 heads, SwiGLU 10752, packed seq 13248 = "
            "text 256 + audio 2x256 + video 8x30x52 (t2va, 2 timesteps, sigma_v 0.5)")


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", default="b200", choices=["b200", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-rows", type=int, default=128)
    p.add_argument("--workload", default="block", choices=["block", "stack", "image", "siglip", "tiny"],
                   help="block (default) prints the benchmark line; the others print one JSON line "
                        "each for the remaining workloads (stack: 50 blocks + heads, image: 50 "
                        "blocks, siglip: one encoder layer x 32 images, tiny: fp32 block)")
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
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


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
def measured_traffic(profile: str, source: str):
    """DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one
    attention step recorded in a profiles/ summary, or None when the kernel
    source has changed since that capture (the summary carries the source's
    sha256)."""
    import hashlib
    import re
    try:
        text = open(os.path.join(ROOT, "profiles", profile)).read()
        m = re.search(r"traffic_bytes_per_step:\s*(\d+)\s+source_sha256:\s*([0-9a-f]{64})", text)
        digest = hashlib.sha256(open(os.path.join(ROOT, source), "rb").read()).hexdigest()
        if m and m.group(2) == digest:
            return int(m.group(1))
    except OSError:
        pass
    return None


# ------------------------------------------------------- algorithmic work
def block_flops(n, H=2688, I=2688, F=10752):
    gemm = {"qkv gemm": 2.0 * n * H * 3 * I, "out gemm": 2.0 * n * I * H,
            "fc1 gemm": 2.0 * n * H * 2 * F, "fc2 gemm": 2.0 * n * F * H}
    gemm["attention"] = 4.0 * n * n * I
    return gemm


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

    # ---- device-timed region
    api.prof_reset()
    api.prof_enable(True)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = api.launch_count()
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    launches = api.launch_count() - launches0
    barrier()
    api.prof_enable(False)
    ms = e0.elapsed_time(e1)
    phases, nblocks = api.prof_collect()
    api.device_status()
    ms_max = max_over_ranks(ms, device, world)

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
    e2e_steps = max(10, args.steps // 4)
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
    # dominant kernel from the per-phase device times (nblocks blocks)
    per_launch = {k: v / max(1, nblocks) for k, v in phases.items() if v > 0}
    dom = max(("attention", "qkv gemm", "out gemm", "fc1 gemm", "fc2 gemm"),
              key=lambda k: per_launch.get(k, 0.0))
    traffic = None
    if dom == "attention":
        traffic = measured_traffic("attn2_block_13248.md",
                                   "packed_multimodal_diffusion_b200/csrc/attn2_tc.cuh")
    peaks = load_peaks()
    achieved = flops[dom] / (per_launch[dom] / 1e3) / 1e12
    peak = peaks["bf16_tflops_sustained"]
    clocks = clk.summary()
    total_flop = sum(flops.values())
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "n_tokens": n, "hidden": 2688, "heads": 21, "head_dim": 128,
                   "ffn": 10752, "timesteps": 2,
                   "l2": "inputs larger than L2 (x 142 MB fp32, weights 231 MB bf16), no flush",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "tflops_per_s": total_flop / (step_ms / 1e3) / 1e12,
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"{peaks['source']} bf16 sustained (MEASURED_PEAKS.json)",
                     "traffic": traffic,
                     "traffic_unit": ("bytes per attention step (whole-unit launch, split-tail launch and "
                                      "merge when the last wave is split)" if dom == "attention"
                                      else "bytes/launch"),
                     "algorithmic_bytes": 2 * n * 3 * 2688 + 2 * n * 2688},
        "phases_ms_per_block": {k: round(v / max(1, nblocks), 4) for k, v in phases.items()},
        "phase_frac_of_peak": {k: round(flops[k] / (per_launch[k] / 1e3) / 1e12 / peak, 4)
                               for k in flops if k in per_launch},
        "e2e": {"value": job_throughput(world, n, e2e_steps, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": int(W["x0"].numel() * 4 + W["pos_d"].numel() * 4),
                "d2h_bytes_per_step": int(W["x0"].numel() * 4)},
        "gpu_launches": launches,
        "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                   "reasons": clocks["reasons"], "samples": clocks["samples"]},
    }
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(args.cpu_rows)
    print(json.dumps(line), flush=True)


# -------------------------------------------------------------- CPU oracle
class OracleSample:
    """The oracle on a bounded sample of the block workload: k and v for all
    tokens (attention reads every key) plus `rows` query rows through the
    whole block.  Inputs are generated once; run() times one sample."""

    def __init__(self, rows: int):
        import numpy as np

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
        self.rows_of = O.token_rows(L["segments"], slot, self.n)
        self.sample = np.linspace(0, self.n - 1, max(2, rows)).astype(int)
        try:
            from threadpoolctl import threadpool_info
            self.cores = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
        except Exception:
            self.cores = os.cpu_count()

    def _block(self, rows):
        O, c, p = self.O, self.c, self.p
        mods = O.block_mods(p["adaln_w"], p["adaln_b"], p["adaln_table"], self.ts, c.hidden)
        O.block_forward(p, self.x, mods, self.rows_of, self.L["pos"], c.dims(), sample_rows=rows)

    def calibrate(self, rows: int = 192, reps: int = 2):
        """Per-row cost of the block (attention over all keys, projections,
        FFN): the difference between a `rows`-row and a 1-row run, each the
        best of `reps`.  Both runs share the fixed cost of k and v for all
        tokens (seconds on the host), so the row count must be large enough
        for the marginal cost to stand well above that cost's run-to-run
        noise."""
        import numpy as np
        big = np.linspace(0, self.n - 1, rows).astype(int)

        def best(r):
            ts = []
            for _ in range(reps):
                t0 = time.perf_counter()
                self._block(r)
                ts.append(time.perf_counter() - t0)
            return min(ts)

        t_one = best(self.sample[:1])
        t_big = best(big)
        self.t_row = max(0.0, (t_big - t_one) / (len(big) - 1))
        self.calib_rows = len(big)

    def run(self):
        """Time one sample; -> (seconds, extrapolated full-block seconds)."""
        if not hasattr(self, "t_row"):
            self.calibrate()
        t0 = time.perf_counter()
        self._block(self.sample)
        t_s = time.perf_counter() - t0
        return t_s, t_s + (self.n - len(self.sample)) * self.t_row

    def describe(self, t_s, t_full):
        return (f"block workload: k/v for all {self.n} tokens + {len(self.sample)} sampled query "
                f"rows through the whole block ({t_s:.2f} s); full {self.n}-row block "
                f"extrapolated with the per-row cost measured between 1 and "
                f"{self.calib_rows} rows, best of 2 ({t_full:.1f} s)")


def cpu_baseline(rows_sample):
    o = OracleSample(rows_sample)
    t_s, t_full = o.run()
    return {"value": N_TOKENS / t_full, "unit": UNIT, "cores": o.cores, "kind": "oracle",
            "sample": o.describe(t_s, t_full)}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    o = OracleSample(max(2, min(args.cpu_rows, 64)))
    fulls, samples = [], []
    for i in range(args.warmup + args.steps):
        t_s, t_full = o.run()
        if i >= args.warmup:
            fulls.append(t_full)
            samples.append(t_s)
    t_full = statistics.mean(fulls)
    value = N_TOKENS / t_full
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * t_full, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": WORKLOAD, "n_tokens": N_TOKENS},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": o.cores, "kind": "oracle",
                             "sample": o.describe(statistics.mean(samples), t_full)},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------- other workloads
def _time(fn, steps, warmup):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def run_workload(args):
    """One JSON line for the stack, image, SigLIP or tiny workload (device-timed
    with CUDA events, weights generated on the device from the seeded streams,
    per-phase profile over the timed steps)."""
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
        api.device_status()
        rows = c.batch * c.seq
        flop = 2.0 * rows * c.hidden * (3 * c.hidden + c.hidden + 2 * c.mlp) + 4.0 * c.batch * c.seq ** 2 * c.hidden
        line.update(metric="SigLIP encoder layer time (bf16, 1 B200)", value=ms, unit="ms/layer",
                    higher_is_better=False, dtype="bf16", tokens_per_s=rows / (ms / 1e3),
                    tflops_per_s=flop / (ms / 1e3) / 1e12,
                    config={"workload": "SigLIP layer: 32 images x 1024 tokens, hidden 768, 12x64 heads, "
                                        "MLP 3072 tanh-GELU, LayerNorm pre-norm"},
                    context="the pages quote 61.9 ms/layer for batch 1 on an unnamed CPU")
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

    api.prof_reset()
    api.prof_enable(True)
    ms = _time(step, steps, warmup)
    api.prof_enable(False)
    phases, nblocks = api.prof_collect()
    api.device_status()
    flops = block_flops(n, c.hidden, c.heads * c.head_dim, c.ffn)
    per_block = {k: v / max(1, nblocks) for k, v in phases.items() if v > 0}
    peak = peaks["bf16_tflops_sustained"]
    line.update(metric=f"{args.workload} forward time (1 B200)", value=ms, unit="ms/forward",
                higher_is_better=False, dtype="fp32/tf32" if c.act_dtype == torch.float32 else "bf16",
                n_tokens=n, n_blocks=c.n_blocks, heads=bool(heads),
                tokens_per_s_per_block=n * c.n_blocks / (ms / 1e3),
                tflops_per_s=c.n_blocks * sum(flops.values()) / (ms / 1e3) / 1e12,
                phases_ms_per_block={k: round(v, 4) for k, v in per_block.items()},
                phase_frac_of_peak={k: round(flops[k] / (per_block[k] / 1e3) / 1e12 / peak, 4)
                                    for k in flops if k in per_block},
                config={"workload": f"{c.name}: n {n}, hidden {c.hidden}, {c.heads}x{c.head_dim} heads, "
                                    f"SwiGLU {c.ffn}, {c.n_blocks} blocks" + (", output heads" if heads else "")})
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.workload != "block":
        run_workload(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
