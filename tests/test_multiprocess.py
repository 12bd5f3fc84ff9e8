"""The N > 1 path on CPU: world-size-2 `gloo` process groups.

The forward shards by token with replicated weights (each rank runs its own
replica of the step), so the only collectives are the barrier around the
timed region and the max over ranks of its time.  These tests run those
steps with two CPU processes, and the reference arm under a two-rank
`torch.distributed.run` launch (rank 0 alone times the oracle and prints the
line; the other rank exits 0 without work).
"""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, results) -> None:
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.argv = ["bench.py"]
    import bench

    d = bench.Dist(world, backend="gloo")
    d.barrier()
    # each rank's "time": the job's time is the slowest rank's
    m = d.max(float(10 * (rank + 1)))
    d.barrier()
    results[rank] = (d.world, d.rank, m)
    d.close()


def test_two_rank_barrier_and_max_over_ranks():
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, 2, port, results)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=240)
            assert p.exitcode == 0
        assert dict(results) == {0: (2, 0, 20.0), 1: (2, 1, 20.0)}


def test_reference_arm_under_two_rank_launch_prints_one_line():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "tiny"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 1 and d["value"] > 0
    assert d["e2e"]["value"] == d["value"] and d["cpu_baseline"]["kind"] == "oracle"
