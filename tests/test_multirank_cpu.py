"""The bench's multi-rank plumbing on the host (world_size 2, gloo): timings are
reduced to the slowest rank's, the barrier works without a GPU, and the
reference arm under torchrun is printed by rank 0 alone with every rank
exiting 0.  The data path has no collective (replicas only), so these host
steps are the whole multi-rank logic."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench._barrier(world, torch)
        got = bench._max_over_ranks(1.5 + rank, world, torch)
        same = bench._max_over_ranks(7.0, world, torch)
        out[rank] = (got, same)
        bench._barrier(world, torch)
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_and_barrier_on_gloo():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res == {0: (2.5, 7.0), 1: (2.5, 7.0)}


def test_single_rank_needs_no_process_group():
    assert bench._max_over_ranks(3.25, 1, torch) == 3.25


def test_reference_arm_under_torchrun_prints_once():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr",
           "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3", "--ref-seconds", "2"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
