"""bench.py's multi-rank path on the CPU: two gloo ranks.

Under torchrun every rank runs its own replica of the workload; the only
cross-rank steps are the barrier around the timed region and the max over
ranks of the device time.  These tests run those helpers on two gloo
processes, and the reference arm under torchrun (rank 0 alone times the
oracle and prints one line, the other rank exits 0 without work).
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch

    import bench
    d = bench.init_dist(world, "gloo")
    dev = torch.device("cpu")
    bench.barrier(d, dev)
    got = bench.max_over_ranks(10.0 * (rank + 1), d, dev)
    bench.barrier(d, dev)
    d.destroy_process_group()
    q.put((rank, got))


def test_max_over_ranks_on_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert results == {0: 20.0, 1: 20.0}


def test_single_rank_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import torch

    import bench
    assert bench.init_dist(1, "gloo") is None
    assert bench.max_over_ranks(3.5, None, torch.device("cpu")) == 3.5
    bench.barrier(None, torch.device("cpu"))


def test_reference_arm_under_torchrun_prints_one_line():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--workload", "tiny_16x16_f32", "--steps", "1", "--warmup", "3",
           "--gpus", "2"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
