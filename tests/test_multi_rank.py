"""The multi-replica bench plumbing on CPU: two gloo ranks (CPU only).

The decode path shards by sequence with no exchange, so the only cross-rank
steps are the timing barrier and the max / sum reductions of the report.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        times = [10.0 + rank, 20.0 - rank]
        amounts = [100.0 * (rank + 1), 1.0]
        res = bench.reduce_over_ranks(dist, torch.device("cpu"), times, amounts)
        out[rank] = res
        out[f"seed{rank}"] = bench.rank_seed(4, rank)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_like_the_bench():
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:    # no fork of a threaded process
        out = mgr.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    for r in (0, 1):
        assert res[r] == [11.0, 20.0, 300.0, 2.0]       # max of times, sum of amounts
    assert res["seed0"] != res["seed1"]                   # each replica has its own batch


def test_single_rank_reduce_is_identity():
    import bench
    assert bench.reduce_over_ranks(None, torch.device("cpu"), [3.0], [4.0, 5.0]) == [3.0, 4.0, 5.0]


def test_reference_arm_prints_on_rank_zero_only():
    """`bench.py --impl reference` under N ranks: rank 0 times the oracle and
    prints one JSON line; every other rank exits 0 without work."""
    import json
    import subprocess
    import sys

    from tests.conftest import ROOT
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--reference-seqs", "2", "--workload", "2"]
    outs = {}
    for rank in (0, 1):
        env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2")
        r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
        assert r.returncode == 0, r.stderr
        outs[rank] = [l for l in r.stdout.splitlines() if l.strip()]
    assert outs[1] == []
    assert len(outs[0]) == 1
    line = json.loads(outs[0][0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
