"""The N > 1 path of bench.py, as world_size-2 gloo ranks on the CPU.

bench.py runs one process per GPU: each rank streams its own block of
decode problems, the ranks meet only at the barriers around the timed
region, and the reported time is the maximum over ranks.  Checked here
without a GPU: the barrier and the max-over-ranks reduction with two real
gloo ranks, the disjointness of the ranks' problem blocks, and the
reference arm under torchrun (rank 0 prints the one JSON line, the other
rank exits 0 without work).
"""
from __future__ import annotations

import json
import multiprocessing as mp
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        got = bench.max_over_ranks(1.5 + rank, world, device="cpu")
        bench.barrier(world)
        q.put((rank, got, bench.dist_env()))
    finally:
        dist.destroy_process_group()


def test_barrier_and_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[1] for g in got] == [2.5, 2.5]          # every rank reports the slowest rank's time
    assert [g[2][:2] for g in got] == [(0, 2), (1, 2)]


def test_rank_problem_blocks_are_disjoint():
    sys.path.insert(0, ROOT)
    import bench
    world = 8
    seeds = [bench.rank_pair_seeds(r) for r in range(world)]
    flat = [x for blk in seeds for x in blk]
    assert len(flat) == len(set(flat)) == world * bench.N_PAIRS
    assert sorted(flat) == list(range(world * bench.N_PAIRS))
    assert seeds[0] == list(range(bench.N_PAIRS))     # rank 0 runs the single-GPU workload


@pytest.mark.slow
def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "1"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1                             # rank 0 alone prints
    out = json.loads(lines[0])
    assert out["impl"] == "reference" and out["n_gpus"] == 2 and out["value"] > 0
    assert out["cpu_baseline"]["kind"] == "oracle"
