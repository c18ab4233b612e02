"""Multi-process host logic of the benchmark on CPU (gloo, world size 2).

bench.py --gpus N runs one independent layer call per rank (replicas: every
rank routes its own token batch, experts replicated, no collective on the data
path), takes the max of the per-rank device times and prints from rank 0 only.
These tests run that plumbing with two gloo ranks on the CPU.
"""
import json
import os
import socket
import subprocess
import sys
from pathlib import Path

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parent.parent


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, str(ROOT))
    import bench
    from sparse_mixture_experts_fp32_b200 import synth
    bench.init_dist(world, "gloo")
    wl = synth.WORKLOADS["base8"]
    t = bench.max_over_ranks(10.0 * (rank + 1), world, "cpu")
    seed = bench.rank_seed(wl, rank)
    x = synth.activations(wl, seed=seed, T=8)
    seeds = [None] * world
    dist.all_gather_object(seeds, (seed, x[0, :4].tolist()))
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, t, seeds))


def test_max_over_ranks_and_distinct_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, seeds in res:
        assert t == 20.0  # the slowest rank's time
        assert seeds[0][0] != seeds[1][0] and seeds[0][1] != seeds[1][1]
    assert {r for r, _, _ in res} == {0, 1}


def test_reference_arm_prints_once_under_torchrun(tmp_path):
    """`bench.py --impl reference` under a 2-rank launch: rank 0 times the
    oracle and prints one JSON line, rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}", str(ROOT / "bench.py"), "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "tiny_fp32", "--cpu-budget", "1"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["config"]["workload"] == "tiny_fp32"
