"""Multi-rank host logic of the benchmark on CPU: two gloo ranks (world size 2).

The Muon step itself has no exchange between ranks: N GPUs run N replicas (weak
scaling), and the only collective is the max-over-ranks reduction of the timing.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        r, w, lr = bench.dist_env()
        ms_local = 100.0 + 25.0 * rank          # rank 1 is the slow one
        ms_max = bench.max_over_ranks(ms_local, w, torch.device("cpu"))
        value = bench.replica_throughput(2e12, 10, w, ms_max)
        out[rank] = (r, w, lr, ms_max, value)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_weak_scaling_value():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0][:3] == (0, 2, 0) and out[1][:3] == (1, 2, 1)
    for r in range(world):
        assert out[r][3] == 125.0                       # max over ranks
        # 2 TFLOP per step x 10 steps x 2 replicas / 0.125 s = 320 TFLOP/s
        assert out[r][4] == pytest.approx(320.0)


def test_single_process_defaults():
    old = {k: os.environ.pop(k, None) for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    try:
        assert bench.dist_env() == (0, 1, 0)
        assert bench.max_over_ranks(7.5, 1, torch.device("cpu")) == 7.5
        assert bench.replica_throughput(1e12, 4, 1, 1000.0) == pytest.approx(4.0)
    finally:
        for k, v in old.items():
            if v is not None:
                os.environ[k] = v


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
