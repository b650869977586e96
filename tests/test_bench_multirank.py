"""The multi-rank (replica) path of bench.py on CPU with the gloo backend, world size 2.

Decode attention has no exchange step, so N GPUs run N independent replicas: each rank
decodes its own seeded batch, the time is the max over ranks and the value is the
whole-job throughput.  The GPU kernels are not run here; the host logic around them is.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        slowest = bench.max_over_ranks(local_ms, dist, "cpu")
        value = bench.job_throughput(1_000_000_000, world, slowest * 1e-3)
        q.put((rank, slowest, value, bench.rank_seed("8b", rank)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, m0, v0, s0), (r1, m1, v1, s1) = got
    assert m0 == m1 == 15.0, "both ranks see the slowest rank's time"
    assert v0 == v1 == pytest.approx(2 * 1e9 / 15e-3 / 1e9), "value counts both replicas' bytes"
    assert s0 != s1, "replicas decode different batches"


def test_max_over_ranks_without_group_is_identity():
    assert bench.max_over_ranks(3.5) == 3.5


def test_reference_arm_under_torchrun_two_ranks():
    """`--impl reference` under torchrun: rank 0 alone runs and prints one line, rank 1 exits 0."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--config", "tiny",
           "--ref-seconds", "1"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
