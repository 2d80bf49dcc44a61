"""The multi-rank path of bench.py on CPU: two gloo ranks.

Each GPU rank runs its own batch of tokens against a replica of the layer
(data parallel over tokens, no collective on the data path); the job's time
is the slowest rank's device time and its throughput is all ranks' work over
that time.  These checks run the aggregation and the rank-0-only reference
arm under a real two-process gloo group.
"""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [2.0, 3.5][rank]            # the second rank is slower
        ms = bench.max_over_ranks(local_ms, world)
        tops = bench.whole_job_tops(1e12, ms, world)
        q.put((rank, ms, tops))
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation_takes_slowest_rank():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for _, ms, tops in res:
        assert ms == 3.5
        assert tops == pytest.approx(2 * 1e12 / 3.5e-3 / 1e12)


def test_single_rank_aggregation_is_identity():
    import bench
    assert bench.max_over_ranks(1.25, 1) == 1.25
    assert bench.whole_job_tops(2e12, 1.0, 1) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import argparse
    import bench
    import workloads
    args = argparse.Namespace(steps=1, warmup=0, ref_rows=1, low="int4", bank=16, high=1)
    assert bench.run_reference(args, workloads.TINY, rank=1, world=2) == 0
    assert capsys.readouterr().out == ""


@pytest.mark.parametrize("low", ["int4", "fp8", "mx", "sqf"])
def test_reference_arm_json_line(low):
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--workload",
                          "tiny_64x256x256_o8", "--steps", "2", "--warmup", "3", "--low", low],
                         capture_output=True, text=True, timeout=300, env={**os.environ, "OMP_NUM_THREADS": "2"})
    assert out.returncode == 0, out.stderr
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TOPS" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"] == "tiny_64x256x256_o8" and line["config"]["low_path"] == low
