"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): a job's
time is its slowest rank's, its throughput counts every rank's units, each
rank seeds its own inputs, and the reference arm runs on rank 0 only."""
import argparse
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

_CHILD = r"""
import datetime, json, os, sys
sys.path.insert(0, os.environ["REPO_ROOT"])
import torch.distributed as dist
import bench
rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
try:
    dist.barrier()
    ms = float(os.environ["MY_MS"])
    slowest = bench.max_over_ranks(ms, world)
    print(json.dumps({"rank": rank, "slowest": slowest, "rate": bench.job_rate(world, 200, slowest),
                      "seed": bench.rank_seed(7, rank)}), flush=True)
    dist.barrier()
finally:
    dist.destroy_process_group()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_ranks_time_the_job_by_the_slowest_rank():
    world, port = 2, _free_port()
    per_rank_ms = [12.5, 20.0]
    procs = []
    for rank in range(world):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), REPO_ROOT=ROOT,
                   MY_MS=str(per_rank_ms[rank]))
        procs.append(subprocess.Popen([sys.executable, "-c", _CHILD], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=180)
        assert p.returncode == 0, err
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for o in outs:
        assert o["slowest"] == max(per_rank_ms)
        assert o["rate"] == pytest.approx(world * 200 / (max(per_rank_ms) / 1e3))
    assert outs[0]["seed"] != outs[1]["seed"]


def test_one_rank_is_its_own_slowest():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_rate(1, 100, 50.0) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank_zero_only():
    args = argparse.Namespace(warmup=3, steps=1)
    assert bench.run_reference(args, bench.CONFIGS["decode_32k"], 1, 2) is None
