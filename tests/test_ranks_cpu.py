"""Multi-process paths of the benchmark on CPU (gloo, world size 2).

The layer has no exchange step, so N GPUs run N independent replicas; the
only cross-rank logic is the max-over-ranks timing, the whole-job throughput,
distinct per-rank token batches, and (for the comparison arm) rank 0 alone
doing the work.  These tests run that logic in real process groups without a
GPU.
"""
import importlib.util
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


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = _bench()
        # every rank measured a different duration; all must report the slowest
        ms = b.max_over_ranks(1.0 + rank, dist, torch.device("cpu"))
        seeds = [b.replica_seed(rank, i) for i in range(16)]
        q.put((rank, ms, seeds))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_replica_seeds_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        rank, ms, seeds = q.get(timeout=120)
        got[rank] = (ms, seeds)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert got[0][0] == got[1][0] == 2.0
    assert not set(got[0][1]) & set(got[1][1]), "replicas must process different token batches"


def test_job_throughput_counts_every_rank():
    b = _bench()
    one = b.job_tops(1e12, 10, 1, 10.0)       # 10 steps of 1 TOP on one rank in 10 ms
    assert one == pytest.approx(1000.0)
    # weak scaling: twice the ranks, same per-rank work, same slowest time
    assert b.job_tops(1e12, 10, 2, 10.0) == pytest.approx(2 * one)
    assert b.max_over_ranks(3.5, None, None) == 3.5


def test_reference_arm_two_ranks_rank0_only():
    # the comparison arm under torchrun: rank 0 runs the oracle and prints one
    # line, the other rank exits 0 without work
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--workload", "tiny", "--steps", "2", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
