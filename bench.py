"""Throughput of the PT-Block attention path (GIIM + TCM) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one ptdit_block_attn call over one batch of the workload (default:
the long high-resolution video, 32 x 64 x 64 = 131072 tokens, D = 1152, 16
heads, bf16, proxy ratio (1,16,16), TCM window 2 x 8 x 8), inputs resident in
HBM.  Each step is timed alone with CUDA events on the launching stream.  When
the step's input is larger than twice the L2 (the long video's 302 MB), it
cannot be in L2 when the next step starts; otherwise L2 is flushed (a 256 MiB
write) before every timed step.
Under torchrun every rank runs its own replica of the workload (batch items
are independent, so there is no data-path collective); the job time is the
max over ranks.  Rank 0 prints one JSON line.

--impl reference times the float64 CPU oracle on the host cores instead: each
step runs the oracle's stages on a bounded sample of one batch item (all
proxies, a sample of latent rows for the cross-attention and a sample of
windows for each TCM branch) and extrapolates the whole item's time from it.

Measurement options beyond the default line: --grid F,H,W and --ratio F,H,W
override the workload's token grid and proxy ratio (the long-video ratio
sweep); --dense times the dense comparator instead, one full global
self-attention module (QKV projection, attention over all N tokens, output
projection and residual) per step on the same grid.
"""
from __future__ import annotations

import argparse
import ctypes
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
L2_BYTES = 126 << 20  # B200


def l2_policy(w):
    """(flush before every timed step?, the config's description of it)."""
    zb = w.B * w.N * w.D * (2 if w.dtype == "bf16" else 4)
    if zb > 2 * L2_BYTES:
        return False, (f"inputs larger than L2: z is {zb / 1e6:.0f} MB against 126 MB of L2, "
                       "so no step finds its input there (no flush)")
    return True, "flushed before every timed step (256 MiB write)"

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of the
# dominant kernel, averaged over the launches of one step, from one ncu capture
# of the current kernel source, per workload.  Absent when the kernel changed
# since the capture.
# The captures in profiles/gemm_tc2_dram_traffic_video_32x64x64.md (641.3 MB per
# launch on the long video) and profiles/gemm_tc2_t2i_2048px_qkv_and_oproj.md
# (59.4 MB at 2048 px) predate the whole-warp MMA issuer of gemm_tc2, so they are
# not used here.
TRAFFIC = {
    # profiles/gemm_tc2_dram_traffic_t2i_1024px.md: one step's nine launches, per launch
    "t2i_1024px_64x64_b4": 59.7e6,
}


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


_FIXED = {}


def oracle_sample_step(w, z64, W64, rng, rows=2048, windows=16):
    """One reference step: the oracle's stages on a bounded sample of one batch
    item, and the whole item's time extrapolated from it.

    Every stage runs the oracle as it stands.  Averaging and proxy self-attention
    run in full (their cost does not grow with the sample); the cross-attention
    runs for `rows` random latent rows and each TCM branch for `windows` random
    windows, and their per-row and per-window times are scaled to the whole
    grid.  A branch's fixed cost (the roll and window partition of the whole
    grid) is timed separately, with no window, and added once.
    Returns (extrapolated seconds per item, seconds spent)."""
    import numpy as np

    import oracle as O
    t_start = time.perf_counter()
    z = z64[0]
    t0 = time.perf_counter()
    Pp = O.proxy_self_attention(z, w.grid, w.ratio, W64["psa"], w.heads)
    t_proxy = time.perf_counter() - t0
    r = rng.choice(w.N, size=min(rows, w.N), replace=False)
    t0 = time.perf_counter()
    _ = z[r] + O.multihead_attention(z[r], Pp, W64["cross"], w.heads)
    t_cross = (time.perf_counter() - t0) * w.N / len(r)
    nwin = w.N // w.n
    t_tcm = 0.0
    for shift, m in (((0, 0, 0), "wsa"), (w.shift, "swsa")):
        if (w.name, shift) not in _FIXED:
            t0 = time.perf_counter()
            O.window_self_attention(z, w.grid, w.window, shift, W64[m], w.heads, windows=[])
            _FIXED[(w.name, shift)] = time.perf_counter() - t0
        fixed = _FIXED[(w.name, shift)]
        k = rng.choice(nwin, size=min(windows, nwin), replace=False)
        t0 = time.perf_counter()
        O.window_self_attention(z, w.grid, w.window, shift, W64[m], w.heads, windows=k)
        part = time.perf_counter() - t0
        t_tcm += fixed + max(0.0, part - fixed) * nwin / len(k)
    return t_proxy + t_cross + t_tcm, time.perf_counter() - t_start


def run_reference(args, w):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    import numpy as np
    z, W = host_inputs(w)
    from diffusion_transformer_sparse_b200 import synth
    z64 = [synth.as_f64(z[0])]
    W64 = {m: tuple(synth.as_f64(x) for x in ws) for m, ws in W.items()}
    rng = np.random.default_rng(2024)
    for _ in range(args.warmup):
        oracle_sample_step(w, z64, W64, rng)
    est, spent = [], 0.0
    for _ in range(args.steps):
        t, dt = oracle_sample_step(w, z64, W64, rng)
        est.append(t)
        spent += dt
    total = sum(est)
    value = args.steps * w.N / total
    sample = (f"per step: one of {w.B} batch items of {w.name}; averaging and proxy SA in "
              f"full, cross-attention on 2048 random latent rows, each TCM branch on 16 "
              f"random windows plus its whole-grid roll, scaled to all {w.N} rows and "
              f"{w.N // w.n} windows (extrapolated); {spent / args.steps:.2f} s of CPU work "
              f"per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(w):
    return {"workload": w.name, "B": w.B, "grid": list(w.grid), "D": w.D, "heads": w.heads,
            "ratio": list(w.ratio), "window": list(w.window), "shift": list(w.shift),
            "tokens_per_step": w.B * w.N, "l2": l2_policy(w)[1]}


# ------------------------------------------------------------------ GPU arm
def kernel_work(w, fused=False):
    """Algorithmic work per step of each kernel kind (library timing-hook names):
    (amount, unit, bound).  Averaging and the window cores are HBM-bound and
    count bytes: averaging reads N and writes M rows of D elements; a window
    core reads Q, K and V and writes O, 4 N D elements per launch.  The others
    count FLOP (a multiply-add is 2).  With the fused window kernel, the two
    window branches' Q/K/V projections (6 N D^2 each) and cores count there."""
    e = 2 if w.dtype == "bf16" else 4
    f = flops.block_flops(w.N, w.M, w.n, w.D)
    B = w.B
    work = {
        "average": (B * flops.average_bytes(w.N, w.M, w.D, e), "bytes", "hbm"),
        "gemm": (B * f["proj"], "flop", "tensor"),
        "attn_proxy": (B * f["psa_core"], "flop", "tensor"),
        "attn_cross": (B * f["cross_core"], "flop", "tensor"),
        "attn_window": (B * 2 * 4 * w.N * w.D * e, "bytes", "hbm"),
    }
    if fused:
        qkv = 2 * 6 * w.N * w.D * w.D
        work["gemm"] = (B * (f["proj"] - qkv), "flop", "tensor")
        work["attn_window_fused"] = (B * (qkv + f["wsa_core"] + f["swsa_core"]), "flop", "tensor")
    return work


def run_gpu(args, w):
    import torch

    import diffusion_transformer_sparse_b200 as pt
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    pt.lib()
    if getattr(args, "fused_window", False):
        pt.lib().ptdit_window_fused(1)

    z_host, W_host = host_inputs(w)
    z = z_host.to(dev)
    W = {m: tuple(x.to(dev) for x in ws) for m, ws in W_host.items()}
    shape = pt.make_shape(z, w.grid, w.heads)
    ws = pt.workspace(shape, w.ratio, w.window)
    out = torch.empty_like(z)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(zin=z, zout=out, s=stream):
        pt.ptdit_block_attn(zin, w.grid, w.ratio, w.window, w.shift, W["psa"], W["cross"],
                            W["wsa"], W["swsa"], w.heads, z_out=zout, ws=ws, stream=s)

    do_flush = l2_policy(w)[0]

    def timed(K, fn):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
        for e0, e1 in evs:
            if do_flush:
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

    # per-kernel durations: the same K steps with the library's event hooks on.
    # An event pair around every launch also keeps each kernel from starting its
    # prologue under the previous one's tail (programmatic dependent launch), so
    # the hooked steps run slower than the timed ones (timing_hook_overhead); the
    # per-kernel times are those of kernels that run alone.
    pt.ptdit_timing_enable(64 * args.steps)
    hooked = timed(args.steps, step)
    recs = pt.ptdit_timing_read(64 * args.steps)
    pt.ptdit_timing_enable(0)
    per_kind = {}
    for k, t in recs:
        d = per_kind.setdefault(k, [0, 0.0])
        d[0] += 1
        d[1] += t
    peaks = load_peaks()
    f = flops.block_flops(w.N, w.M, w.n, w.D)
    step_flops = w.B * f["total"]
    work = kernel_work(w, fused="attn_window_fused" in per_kind)
    kernels = {}
    hooked_kernel_ms = sum(v[1] for v in per_kind.values()) / args.steps
    for k, (n, t) in sorted(per_kind.items()):
        kms = t / args.steps
        ent = {"launches_per_step": n / args.steps, "ms_per_step": kms,
               "share": kms / max(1e-9, hooked_kernel_ms)}
        if k in work and kms > 0:
            amount, unit, bound = work[k]
            if unit == "bytes":
                ach = amount / (kms / 1e3) / 1e9
                ent.update({"bound": "hbm", "algorithmic_bytes_per_step": amount,
                            "achieved": ach, "unit": "GB/s", "peak": peaks["hbm"],
                            "frac": ach / peaks["hbm"]})
            else:
                ach = amount / (kms / 1e3) / 1e12
                ent.update({"bound": "tensor", "algorithmic_flop_per_step": amount,
                            "achieved": ach, "unit": "TFLOP/s", "peak": peaks["bf16"],
                            "frac": ach / peaks["bf16"]})
        kernels[k] = ent
    gemm_n, gemm_t = per_kind.get("gemm", [0, 0.0])
    gemm_ms = gemm_t / args.steps
    proj_flops = work["gemm"][0]
    achieved = proj_flops / (gemm_ms / 1e3) / 1e12 if gemm_ms > 0 else None
    peak_note = "measured" if peaks["source"] == "measured" else "fallback"
    traffic = TRAFFIC.get(w.name)
    roofline = {
        "kernel": "gemm_tc2 (QKV and O projections)", "bound": "tensor",
        "achieved": achieved, "peak": peaks["bf16"], "unit": "TFLOP/s",
        "frac": achieved / peaks["bf16"] if achieved else None,
        "traffic": traffic,
        "peak_kind": f"bf16 dense burst, of {peak_note} (each launch is timed alone, "
                     f"well under a second)",
        "frac_of_sustained": achieved / peaks["bf16_sustained"] if achieved else None,
        "launches_per_step": gemm_n / args.steps,
        "flops_per_launch": proj_flops / max(1, gemm_n / args.steps),
        "flops_per_step": proj_flops,
    }
    hook_overhead = sum(hooked) / max(1e-9, sum(ms))

    # end to end through the public call: every step copies its input from pinned
    # host memory and its result back.  Step k's input copy runs on its own
    # stream during step k - 1 and step k's output copy during step k + 1
    # (double-buffered device tensors, ordered by events), so PCIe and the
    # computation overlap the way a serving loop would run them.
    e2e = e2e_pipelined(args.steps, w, z_host, step, dev, stream, dist)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, z_host, W_host, args.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic (seeded N(0,1) latents, Xavier-uniform weights)",
            "config": dict(config_of(w), window_kernels="fused projection + attention"
                           if getattr(args, "fused_window", False) else "projection, then attention"),
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


def e2e_pipelined(K, w, z_host, step, dev, stream, dist):
    """Tokens/s of K steps, each copying its input host -> device and its output
    device -> host, with the copies overlapped with neighbouring steps."""
    import torch
    z_pin = z_host.pin_memory()
    h_out = [torch.empty_like(z_host).pin_memory() for _ in range(2)]
    d_in = [torch.empty(z_host.shape, dtype=z_host.dtype, device=dev) for _ in range(2)]
    d_out = [torch.empty_like(d_in[0]) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def run(K):
        ev = lambda: torch.cuda.Event()
        h2d, comp, d2h = [ev() for _ in range(K)], [ev() for _ in range(K)], [ev() for _ in range(K)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        s_in.wait_event(t0)

        def copy_in(k):
            with torch.cuda.stream(s_in):
                if k >= 2:
                    s_in.wait_event(comp[k - 2])  # step k - 2 has read d_in[k % 2]
                d_in[k % 2].copy_(z_pin, non_blocking=True)
                h2d[k].record(s_in)

        copy_in(0)
        for k in range(K):
            if k + 1 < K:
                copy_in(k + 1)
            stream.wait_event(h2d[k])
            if k >= 2:
                stream.wait_event(d2h[k - 2])  # d_out[k % 2] has been copied out
            step(d_in[k % 2], d_out[k % 2], stream)
            comp[k].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp[k])
                h_out[k % 2].copy_(d_out[k % 2], non_blocking=True)
                d2h[k].record(s_out)
        stream.wait_event(d2h[K - 1])
        t1.record(stream)
        torch.cuda.synchronize(dev)
        return t0.elapsed_time(t1)

    run(2)
    barrier(dist, dev)
    e2e_ms = max_over_ranks(run(K), dist, dev)
    world = dist.get_world_size() if dist is not None else 1
    zbytes = z_host.numel() * z_host.element_size()
    return {"value": world * K * w.B * w.N / (e2e_ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": zbytes, "d2h_bytes_per_step": zbytes,
            "ms_per_step": e2e_ms / K,
            "note": "input and output copies double-buffered on their own streams"}


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


def run_block(args, w, L=120):
    """The complete PT-Block (ptdit_pt_block): GIIM, TCM, text cross-attention over
    L text tokens and the MLP (D -> 4 D -> D), pre-norm residual sub-layers."""
    import torch

    import diffusion_transformer_sparse_b200 as pt
    from diffusion_transformer_sparse_b200 import synth
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    z_host, W_host = host_inputs(w)
    z = z_host.to(dev)
    Dh = 4 * w.D
    bp = synth.block_params(w.D, Dh, w.dtype)
    attn = {m: tuple(x.to(dev) for x in ws) for m, ws in W_host.items()}
    attn["text"] = tuple(x.to(dev) for x in bp["text"])
    norms = {k: tuple(x.to(dev) for x in v) for k, v in bp["norms"].items()}
    mlp_w = tuple(x.to(dev) for x in bp["mlp"])
    text = synth.text_tokens(w.B, L, w.D, w.dtype).to(dev)
    shape = pt.make_shape(z, w.grid, w.heads)
    ws = pt.pt_block_workspace(shape, w.ratio, L, Dh)
    out = torch.empty_like(z)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        pt.ptdit_pt_block(z, w.grid, w.ratio, w.window, w.shift, attn, norms, mlp_w, text,
                          w.heads, z_out=out, ws=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for e0, e1 in evs:
        flush.zero_()
        e0.record(stream)
        step()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = sum(e0.elapsed_time(e1) for e0, e1 in evs) / args.steps
    pt.ptdit_timing_enable(64 * args.steps)
    for _ in range(args.steps):
        flush.zero_()
        step()
    recs = pt.ptdit_timing_read(64 * args.steps)
    pt.ptdit_timing_enable(0)
    per = {}
    for k, t in recs:
        per[k] = per.get(k, 0.0) + t / args.steps
    f = flops.pt_block_flops(w.N, w.M, w.n, w.D, L, Dh)
    print(json.dumps({
        "mode": "pt_block", "metric": "complete PT-Block tokens/s", "unit": UNIT,
        "value": w.B * w.N / (ms / 1e3), "ms_per_step": ms, "steps": args.steps,
        "warmup": args.warmup, "config": dict(config_of(w), text_len=L, mlp_hidden=Dh),
        "tflops": w.B * f["total"] / (ms / 1e3) / 1e12,
        "kernels_ms_per_step": per, "note": "per-kernel times from a second pass with hooks"}),
        flush=True)
    return 0


def run_bwd(args, w, branch=False, train=False):
    """Backward of the block-attention path (ptdit_block_attn_bwd: GIIM recomputed, TCM's
    backward, GIIM's backward), or with branch=True of the shifted-window TCM branch
    alone (ptdit_window_attn_bwd): dL/dz and the weight gradients for a synthetic
    upstream gradient, per step."""
    import torch

    import diffusion_transformer_sparse_b200 as pt
    from diffusion_transformer_sparse_b200 import synth
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    z_host, W_host = host_inputs(w)
    z = z_host.to(dev)
    dout = torch.stack([synth.latent(w.N, w.D, 500 + b, w.dtype) for b in range(w.B)]).to(dev)
    W = {m: tuple(x.to(dev) for x in W_host[m]) for m in ("psa", "cross", "wsa", "swsa")}
    shape = pt.make_shape(z, w.grid, w.heads)
    dz = torch.empty_like(z)
    nmod = 1 if branch else 4
    dw = [tuple(torch.empty(w.D, w.D, dtype=torch.float32, device=dev) for _ in range(4))
          for _ in range(nmod)]
    if branch:
        ws = pt.window_attn_bwd_workspace(shape, w.window)
    elif train:
        ws = pt.train_workspace(z, w.grid, w.ratio, w.window, w.heads)
        zout = torch.empty_like(z)
    else:
        n = pt.lib().ptdit_block_attn_bwd_workspace_bytes(ctypes.byref(shape), pt._i3(w.ratio),
                                                         pt._i3(w.window))
        ws = torch.empty(n, dtype=torch.uint8, device=dev)
    do_flush = l2_policy(w)[0]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    wg = [pt.AttnWgrad(*[x.data_ptr() for x in g]) for g in dw]
    wa = [pt.attn_w(W[m]) for m in ("psa", "cross", "wsa", "swsa")]

    def step():
        if branch:
            pt.ptdit_window_attn_bwd(z, dout, w.grid, w.window, w.shift, W["swsa"], w.heads,
                                     dz_in=dz, dw=dw[0], ws=ws, stream=stream)
            return
        if train:
            args3 = (ctypes.byref(shape), pt._i3(w.ratio), pt._i3(w.window), pt._i3(w.shift),
                     *[ctypes.byref(x) for x in wa], 0, z.data_ptr())
            rc = pt.lib().ptdit_block_attn_fwd_train(*args3, zout.data_ptr(), ws.data_ptr(),
                                                     ws.numel(), stream.cuda_stream)
            if rc == 0:
                rc = pt.lib().ptdit_block_attn_bwd_saved(
                    *args3, dout.data_ptr(), dz.data_ptr(), *[ctypes.byref(x) for x in wg],
                    ws.data_ptr(), ws.numel(), stream.cuda_stream)
            if rc != 0:
                raise pt.PtditError(rc, pt.lib().ptdit_last_error().decode())
            return
        rc = pt.lib().ptdit_block_attn_bwd(
            ctypes.byref(shape), pt._i3(w.ratio), pt._i3(w.window), pt._i3(w.shift),
            *[ctypes.byref(x) for x in wa], 0, z.data_ptr(), dout.data_ptr(), dz.data_ptr(),
            *[ctypes.byref(x) for x in wg], ws.data_ptr(), ws.numel(), stream.cuda_stream)
        if rc != 0:
            raise pt.PtditError(rc, pt.lib().ptdit_last_error().decode())

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    n0 = pt.ptdit_launch_count()
    for e0, e1 in evs:
        if do_flush:
            flush.zero_()
        e0.record(stream)
        step()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    launches = (pt.ptdit_launch_count() - n0) // args.steps
    ms = sum(e0.elapsed_time(e1) for e0, e1 in evs) / args.steps
    pt.ptdit_timing_enable(128 * args.steps)
    for _ in range(args.steps):
        if do_flush:
            flush.zero_()
        step()
    recs = pt.ptdit_timing_read(128 * args.steps)
    pt.ptdit_timing_enable(0)
    per = {}
    for k, t in recs:
        per[k] = per.get(k, 0.0) + t / args.steps
    if branch:
        f = flops.window_bwd_flops(w.N, w.n, w.D)
        metric, mode = "backward of one TCM branch, tokens/s", "window_bwd"
        cores = {"attn_window_bwd": w.B * f["core_bwd"]}
    elif train:
        f = flops.train_step_flops(w.N, w.M, w.n, w.D)
        metric = "training step of the block-attention path (forward keeping its activations, then backward), tokens/s"
        mode = "train_step"
        cores = {"attn_window_bwd": w.B * f["window_core_bwd"],
                 "attn_rows_bwd": w.B * f["rows_core_bwd"]}
    else:
        f = flops.block_bwd_flops(w.N, w.M, w.n, w.D)
        metric, mode = "backward of the block-attention path (GIIM + TCM), tokens/s", "block_bwd"
        cores = {"attn_window_bwd": w.B * f["window_core_bwd"],
                 "attn_rows_bwd": w.B * f["rows_core_bwd"]}
    rate = {k: v / (per[k] / 1e3) / 1e12 for k, v in cores.items() if per.get(k)}
    print(json.dumps({
        "mode": mode, "metric": metric, "unit": UNIT,
        "value": w.B * w.N / (ms / 1e3), "ms_per_step": ms, "steps": args.steps,
        "warmup": args.warmup, "config": dict(config_of(w), l2=l2_policy(w)[1]),
        "tflops": w.B * f["total"] / (ms / 1e3) / 1e12, "flops_per_step": w.B * f["total"],
        "gpu_launches": launches, "kernels_ms_per_step": per, "kernels_tflops": rate,
        "note": "per-kernel times from a second pass with hooks"}), flush=True)
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
    ap.add_argument("--fused-window", action="store_true",
                    help="take the fused window Q/K/V projection + attention kernel "
                         "(ptdit_window_fused(1)) for windows of 128 tokens")
    ap.add_argument("--bwd", action="store_true",
                    help="time the backward of the block-attention path instead")
    ap.add_argument("--train", action="store_true",
                    help="time a training step of the block-attention path: the forward that "
                         "keeps its activations, then the backward from them")
    ap.add_argument("--bwd-branch", action="store_true",
                    help="time the backward of the shifted-window TCM branch alone instead")
    ap.add_argument("--block", action="store_true",
                    help="time the complete PT-Block (norms, text cross-attention, MLP) instead")
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
    if args.bwd or args.bwd_branch or args.train:
        return run_bwd(args, w, branch=args.bwd_branch, train=args.train)
    if args.block:
        return run_block(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
