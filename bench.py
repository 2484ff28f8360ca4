"""Throughput of the PT-Block attention path (GIIM + TCM) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one ptdit_block_attn call over one batch of the workload (default:
the 1024px text-to-image grid, 4 x 64 x 64 tokens, D = 1152, 16 heads, bf16),
inputs resident in HBM.  L2 is flushed (a 256 MiB write) before every timed
step and each step is timed alone with CUDA events on the launching stream.
Under torchrun every rank runs its own replica of the workload (batch items
are independent, so there is no data-path collective); the job time is the
max over ranks.  Rank 0 prints one JSON line.

--impl reference times the float64 CPU oracle on the host cores instead, one
batch item per step.

Measurement options beyond the default line: --grid F,H,W and --ratio F,H,W
override the workload's token grid and proxy ratio (the long-video ratio
sweep); --dense times the dense comparator instead, one full global
self-attention module (QKV projection, attention over all N tokens, output
projection and residual) per step on the same grid.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from diffusion_transformer_sparse_b200 import configs, flops  # noqa: E402

METRIC = "PT-Block attention tokens/s and TFLOP/s (bf16, 1 B200) vs tensor/HBM roofline"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 256 << 20

# DRAM bytes per launch of the dominant kernel from one ncu capture of the
# current kernel source (None when the kernel changed since the capture).
TRAFFIC = {}


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            p = json.load(fh)
        return {"hbm": p["hbm_gbs"], "bf16": p["bf16_tflops"],
                "bf16_sustained": p["bf16_tflops_sustained"], "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------ distributed plumbing
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    if world <= 1:
        return None
    import datetime

    import torch.distributed as dist
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, dist, device) -> float:
    """Largest x over all ranks (x itself when not distributed)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist, device):
    if dist is None:
        return
    import torch
    dist.barrier(device_ids=[device.index] if device.type == "cuda" else None)


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as fh:
            for line in fh:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        busy = [s for s in sm if s > 0.5 * max(sm)] if sm else []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------------ CPU oracle
def oracle_step(w, z64, W64, b):
    import oracle as O
    return O.block_attn(z64[b], w.grid, w.ratio, w.window, w.shift, W64["psa"], W64["cross"],
                        W64["wsa"], W64["swsa"], w.heads)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def host_inputs(w):
    from diffusion_transformer_sparse_b200 import synth
    z = synth.latents(w.B, w.N, w.D, w.dtype)
    W = synth.weights(w.D, w.dtype)
    return z, W


def cpu_baseline(w, z, W, min_seconds=10.0, max_items=16):
    """The oracle, as it stands, on whole batch items of the workload, cycling
    through the batch until at least `min_seconds` of CPU work are done."""
    from diffusion_transformer_sparse_b200 import synth
    z64 = [synth.as_f64(z[b]) for b in range(w.B)]
    W64 = {m: tuple(synth.as_f64(x) for x in ws) for m, ws in W.items()}
    t0 = time.perf_counter()
    items = 0
    while items < max_items and (items < 1 or time.perf_counter() - t0 < min_seconds):
        oracle_step(w, z64, W64, items % w.B)
        items += 1
    dt = time.perf_counter() - t0
    return {"value": items * w.N / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{items} batch items ({items * w.N} tokens) of {w.name}, full "
                      f"block_attn in float64, {dt:.1f} s"}


def run_reference(args, w):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    z, W = host_inputs(w)
    from diffusion_transformer_sparse_b200 import synth
    z64 = [synth.as_f64(z[0])]
    W64 = {m: tuple(synth.as_f64(x) for x in ws) for m, ws in W.items()}
    for _ in range(args.warmup):
        oracle_step(w, z64, W64, 0)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_step(w, z64, W64, 0)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = args.steps * w.N / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"one of {w.B} batch items of {w.name} per step, full "
                                   "block_attn in float64"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(w):
    return {"workload": w.name, "B": w.B, "grid": list(w.grid), "D": w.D, "heads": w.heads,
            "ratio": list(w.ratio), "window": list(w.window), "shift": list(w.shift),
            "tokens_per_step": w.B * w.N, "l2": "flushed before every timed step (256 MiB write)"}


# ------------------------------------------------------------------ GPU arm
def run_gpu(args, w):
    import torch

    import diffusion_transformer_sparse_b200 as pt
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    pt.lib()

    z_host, W_host = host_inputs(w)
    z = z_host.to(dev)
    W = {m: tuple(x.to(dev) for x in ws) for m, ws in W_host.items()}
    shape = pt.make_shape(z, w.grid, w.heads)
    ws = pt.workspace(shape, w.ratio, w.window)
    out = torch.empty_like(z)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(zin=z, zout=out):
        pt.ptdit_block_attn(zin, w.grid, w.ratio, w.window, w.shift, W["psa"], W["cross"],
                            W["wsa"], W["swsa"], w.heads, z_out=zout, ws=ws, stream=stream)

    def timed(K, fn):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
        for e0, e1 in evs:
            flush.zero_()
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        return [e0.elapsed_time(e1) for e0, e1 in evs]

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)

    # timed region: device time of K steps, max over ranks
    barrier(dist, dev)
    torch.cuda.synchronize(dev)
    launches0 = pt.ptdit_launch_count()
    with ClockSampler(local if "CUDA_VISIBLE_DEVICES" not in os.environ else
                      int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local])) as clk:
        ms = timed(args.steps, step)
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    launches = pt.ptdit_launch_count() - launches0
    total_ms = max_over_ranks(sum(ms), dist, dev)
    value = world * args.steps * w.B * w.N / (total_ms / 1e3)
    ms_step = total_ms / args.steps

    if args.kernels_only:
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                              "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                              "config": config_of(w), "gpu_launches": launches,
                              "note": "--kernels-only: timed region only, for profiling"}),
                  flush=True)
        if dist is not None:
            dist.destroy_process_group()
        return 0

    # per-kernel durations: the same K steps with the library's event hooks on
    pt.ptdit_timing_enable(64 * args.steps)
    hooked = timed(args.steps, step)
    recs = pt.ptdit_timing_read(64 * args.steps)
    pt.ptdit_timing_enable(0)
    per_kind = {}
    for k, t in recs:
        d = per_kind.setdefault(k, [0, 0.0])
        d[0] += 1
        d[1] += t
    f = flops.block_flops(w.N, w.M, w.n, w.D)
    peaks = load_peaks()
    step_flops = w.B * f["total"]
    gemm_ms = per_kind.get("gemm", [0, 0.0])[1] / args.steps
    gemm_launches = per_kind.get("gemm", [0, 0.0])[0] / args.steps
    proj_flops = w.B * f["proj"]
    achieved = proj_flops / (gemm_ms / 1e3) / 1e12 if gemm_ms > 0 else None
    roofline = {
        "kernel": "gemm (QKV and O projections)", "bound": "tensor",
        "achieved": achieved, "peak": peaks["bf16_sustained"], "unit": "TFLOP/s",
        "frac": achieved / peaks["bf16_sustained"] if achieved else None,
        "traffic": TRAFFIC.get("gemm"),
        "peak_kind": f"bf16 sustained, {peaks['source']}",
        "launches_per_step": gemm_launches,
        "flops_per_step": proj_flops,
    }
    kernels = {k: {"launches_per_step": v[0] / args.steps, "ms_per_step": v[1] / args.steps,
                   "share": v[1] / max(1e-9, sum(x[1] for x in per_kind.values()))}
               for k, v in sorted(per_kind.items())}
    hook_overhead = sum(hooked) / max(1e-9, sum(ms))

    # end to end through the public call with pinned host buffers
    z_pin = z_host.pin_memory()
    out_pin = torch.empty_like(z_host).pin_memory()

    def e2e_step():
        z.copy_(z_pin, non_blocking=True)
        step()
        out_pin.copy_(out, non_blocking=True)

    for _ in range(2):
        e2e_step()
    barrier(dist, dev)
    e2e_ms = max_over_ranks(sum(timed(args.steps, e2e_step)), dist, dev)
    zbytes = z.numel() * z.element_size()
    e2e = {"value": world * args.steps * w.B * w.N / (e2e_ms / 1e3), "unit": UNIT,
           "h2d_bytes_per_step": zbytes, "d2h_bytes_per_step": zbytes}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, z_host, W_host, args.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic (seeded N(0,1) latents, Xavier-uniform weights)",
            "config": config_of(w),
            "tflops": step_flops / (ms_step / 1e3) / 1e12,
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk.summary(),
            "kernels": kernels,
            "timing_hook_overhead": hook_overhead,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def run_dense(args, w):
    """The dense comparator: ptdit_full_attn over the workload's grid."""
    import torch

    import diffusion_transformer_sparse_b200 as pt
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    z_host, W_host = host_inputs(w)
    z = z_host.to(dev)
    Wd = tuple(x.to(dev) for x in W_host["wsa"])
    shape = pt.make_shape(z, w.grid, w.heads)
    ws = pt.workspace(shape, None, None)
    out = torch.empty_like(z)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        pt.ptdit_full_attn(z, w.grid, Wd, w.heads, z_out=out, ws=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    pt.ptdit_timing_enable(8 * args.steps)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for e0, e1 in evs:
        flush.zero_()
        e0.record(stream)
        step()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    recs = pt.ptdit_timing_read(8 * args.steps)
    pt.ptdit_timing_enable(0)
    ms = sum(e0.elapsed_time(e1) for e0, e1 in evs) / args.steps
    core_ms = sum(t for k, t in recs if k == "attn_dense") / args.steps
    f = flops.dense_flops(w.N, w.D)
    print(json.dumps({
        "mode": "dense", "metric": "dense global self-attention module tokens/s", "unit": UNIT,
        "value": w.B * w.N / (ms / 1e3), "ms_per_step": ms, "steps": args.steps,
        "warmup": args.warmup, "config": config_of(w),
        "tflops": w.B * f["total"] / (ms / 1e3) / 1e12,
        "core_ms": core_ms, "core_tflops": w.B * f["core"] / (core_ms / 1e3) / 1e12,
        "note": "timing hooks on (one event pair per launch)"}), flush=True)
    return 0


def parse3(text):
    v = tuple(int(x) for x in text.split(","))
    if len(v) != 3:
        raise argparse.ArgumentTypeError("expected three comma-separated integers")
    return v


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=configs.HEADLINE, choices=configs.ORDER)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernels-only", action="store_true",
                    help="stop after the timed region (no hook, e2e or CPU passes): for ncu")
    ap.add_argument("--grid", type=parse3, help="override the token grid F,H,W")
    ap.add_argument("--ratio", type=parse3, help="override the proxy ratio F,H,W")
    ap.add_argument("--dense", action="store_true",
                    help="time the dense comparator (full global self-attention) instead")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    w = configs.WORKLOADS[args.workload]
    if args.grid or args.ratio:
        g, r = args.grid or w.grid, args.ratio or w.ratio
        w = w.with_(grid=g, ratio=r,
                    name=f"{w.name}@grid{'x'.join(map(str, g))}_ratio{'x'.join(map(str, r))}")
    if args.impl == "reference":
        return run_reference(args, w)
    if args.dense:
        return run_dense(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
