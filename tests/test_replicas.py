"""The multi-GPU path (independent replicas) on CPU: world_size-2 gloo ranks.

The runtime has no exchange step between GPUs; what the N > 1 path adds is
the timing protocol (barriers, the maximum of the elapsed times over ranks,
the whole-job rate) and rank 0 alone printing. Both are exercised here with
gloo process groups on 127.0.0.1, and bench.py's reference arm runs under
torchrun with two ranks.
"""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

from persistent_execution_b200 import replicas as R

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), LOCAL_RANK=str(rank),
                      WORLD_SIZE=str(world))
    r = R.init("gloo", timeout_s=60)
    try:
        R.barrier(r)
        elapsed = 1.0 + rank  # the slower rank takes 2 s
        m = R.max_over_ranks(r, elapsed)
        rate = R.job_throughput(1000, r, m)
        R.barrier(r)
        q.put((rank, m, rate))
    finally:
        R.finalize(r)


def test_max_over_ranks_and_job_rate_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(i, world, port, q)) for i in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, m, rate in got:
        assert m == 2.0  # every rank sees the slowest rank's time
        assert rate == 1000 * 2 / 2.0  # units of all ranks over that time


def test_single_process_needs_no_group():
    r = R.Ranks(0, 0, 1)
    assert R.max_over_ranks(r, 3.5) == 3.5
    assert R.job_throughput(10, r, 2.0) == 5.0
    R.barrier(r)
    R.finalize(r)


def test_bench_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--config", "1", "--steps", "2", "--warmup", "1", "--ref-sample", "50"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["n_gpus"] == 2 and j["value"] > 0
    assert j["cpu_baseline"]["kind"] == "oracle" and j["e2e"]["h2d_bytes_per_step"] == 0
