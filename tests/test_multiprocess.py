"""Multi-process host logic of the benchmark, on CPU with the gloo backend.

The decode path has no exchange step (every (batch, KV head) is independent),
so N GPUs run N weak-scaled replicas; what is shared across ranks is only the
max-over-ranks reduction of their device times and the job-level figures.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

import bench
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [10.0, 12.5][rank]  # rank 1 is the slowest
        m = bench.max_over_ranks(local_ms, world)
        results[rank] = (m, bench.whole_job_us_per_step(m, steps=5, world=world),
                         bench.replica_seed(1000, rank))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_rank():
    world = 2
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_worker, args=(world, _free_port(), results), nprocs=world, join=True)
        res = dict(results)
    assert res[0][0] == res[1][0] == 12.5
    # 2 ranks x 5 steps of one layer-step each in 12.5 ms: 1250 us per layer-step
    assert res[0][1] == res[1][1] == pytest.approx(12.5e3 / 10)
    assert res[0][2] != res[1][2]


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.whole_job_us_per_step(3.0, 3, 1) == pytest.approx(1000.0)


def test_replicas_draw_different_inputs():
    wl = workloads.get("tiny").with_(S=32)
    a = workloads.keys_block(wl.with_(seed=bench.replica_seed(wl.seed, 0)), 0, 0)
    b = workloads.keys_block(wl.with_(seed=bench.replica_seed(wl.seed, 1)), 0, 0)
    assert not (a == b).all()


def _run_reference(rank, world):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                           "--steps", "2", "--warmup", "1"], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=300)


def test_reference_arm_runs_on_rank0_only():
    r1 = _run_reference(1, 2)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _run_reference(0, 2)
    assert r0.returncode == 0, r0.stderr
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["higher_is_better"] is False and line["value"] > 0
