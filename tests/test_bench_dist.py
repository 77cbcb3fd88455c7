"""The multi-rank host path of bench.py on CPU (gloo, world size 2).

The decode shards as independent replicas with no data-path collective; what
ranks share is the barrier around the timed region and the max/sum reductions
of time and work.  These run here with the gloo backend.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import bench
    r, local, w = bench.dist_setup(world)
    dev = torch.device("cpu")
    bench.barrier(w)
    mx = bench.reduce_max(1.5 + r, w, dev)
    sm = bench.reduce_sum(10.0 * (r + 1), w, dev)
    q.put((r, mx, sm))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_reductions_across_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert got == [(0, 2.5, 30.0), (1, 2.5, 30.0)]


def test_reference_arm_under_torchrun_prints_one_line():
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.join(ROOT, "bench.py"),
           "--gpus", "2", "--impl", "reference", "--workload", "tiny", "--steps", "2",
           "--warmup", "1"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_percentiles_and_roofline_helpers():
    sys.path.insert(0, ROOT)
    import bench
    med, p10, p90 = bench.percentiles(list(range(1, 102)))
    assert (med, p10, p90) == (51, 11, 91)
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 100.0}
    # 1 GB in 2 ms at 1000 GB/s peak: HBM-bound, 500 GB/s achieved, half the peak
    r = bench.roofline_of(1e9, 1e9, 2e-3, peaks)
    assert r["bound"] == "hbm" and abs(r["achieved"] - 500.0) < 1e-9 and abs(r["frac"] - 0.5) < 1e-12
    assert abs(r["bound_us"] - 1000.0) < 1e-6
    # 1 TFLOP in 20 ms at 100 TFLOP/s: tensor-bound (10 ms against 1 ms of bytes)
    r = bench.roofline_of(1e9, 1e12, 2e-2, peaks)
    assert r["bound"] == "tensor" and abs(r["frac"] - 0.5) < 1e-12
