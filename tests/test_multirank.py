"""The multi-GPU path of bench.py on CPU: two gloo ranks.

bench.py runs one process per GPU. Each rank quantizes its own layer (seed + rank), so no data
moves between ranks. The process group only carries the barrier around the timed region and the
max over ranks of the device time. Rank 0 alone prints the JSON line, and the reference arm runs
on rank 0 only. These tests run that host logic with the gloo backend; no GPU is involved.
"""

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


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    import torch.distributed as dist
    w, r, local = bench.dist_env()
    assert (w, r, local) == (world, rank, rank)
    distributed = bench.init_dist(w, local, backend="gloo")
    try:
        assert distributed
        bench.barrier(distributed)
        # the slowest rank's time is the job's time, on every rank
        t = bench.max_over_ranks(10.0 + 5.0 * rank, distributed, torch.device("cpu"))
        wl = bench.rank_workload("linear_512", rank)
        W = bench.workloads.make_weights(wl, device="cpu")
        results[rank] = (t, wl.seed, float(W.double().sum()))
        bench.barrier(distributed)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_distinct_layers():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        results = m.dict()
        mp.spawn(_rank_main, args=(world, port, results), nprocs=world, join=True)
        res = dict(results)
    assert res[0][0] == res[1][0] == 15.0           # max over ranks, seen by both
    assert res[0][1] != res[1][1]                   # one layer per rank: different seeds
    assert res[0][2] != res[1][2]                   # ... and different weights


def test_job_value_is_all_units_over_the_slowest_rank():
    import bench
    # 2 ranks x 10 steps x 45M weights in 120 ms (the max over ranks)
    assert bench.job_value(2, 10, 45_088_768, 120.0) == pytest.approx(2 * 10 * 45_088_768 / 0.120)
    assert bench.job_value(1, 1, 100, 1000.0) == pytest.approx(100.0)


@pytest.mark.timeout(600)
def test_reference_arm_prints_once_under_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "linear_512", "--steps", "1", "--warmup", "3"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1                           # rank 0 alone prints
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
