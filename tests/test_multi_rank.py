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


# ---------------------------------------------------------------- matrix-sharded step (host logic)

from muon_newton_schulz_06_b200 import sharded  # noqa: E402
import oracle  # noqa: E402
import synth  # noqa: E402


def test_lpt_partition_balances_the_llama_set():
    shapes = [(s.rows, s.cols) for s in synth.config_shapes(4)]
    from muon_newton_schulz_06_b200.cost import ns_flops
    for world in (1, 2, 4, 8):
        owner = sharded.partition_lpt(shapes, world)
        assert sorted(set(owner)) == list(range(world))
        loads = [sum(ns_flops([shapes[i]])["algorithmic"] for i in range(len(shapes)) if owner[i] == r)
                 for r in range(world)]
        assert max(loads) / (sum(loads) / world) < 1.03, (world, loads)
    assert sharded.partition_lpt(shapes, 3) == sharded.partition_lpt(shapes, 3)  # deterministic


def test_end_to_end_chunks_cover_the_set_in_balanced_contiguous_runs():
    from muon_newton_schulz_06_b200.cost import contiguous_chunks, ns_flops
    for cfg in (1, 2, 3, 4):
        shapes = [(s.rows, s.cols) for s in synth.config_shapes(cfg)]
        for n in (1, 2, 4, 7):
            b = contiguous_chunks(shapes, n)
            assert len(b) == n and b[0][0] == 0 and b[-1][1] == len(shapes)
            assert all(x[1] == y[0] for x, y in zip(b, b[1:])) and all(e > a for a, e in b)
            work = [ns_flops(shapes[a:e])["algorithmic"] for a, e in b]
            assert max(work) / (sum(work) / n) < 1.25, (cfg, n, work)
    # fewer matrices than chunks, one dominant matrix, empty list
    assert contiguous_chunks([(4, 4)] * 3, 4) == [(0, 1), (1, 2), (2, 3)]
    assert contiguous_chunks([(100, 100), (4, 4), (4, 4), (4, 4)], 4) == [(0, 1), (1, 2), (2, 3), (3, 4)]
    assert contiguous_chunks([], 4) == []


def _oracle_step(params, grads, moms, lr=0.02, momentum=0.95, **kw):
    """Stands in for the CUDA step on CPU: the float64 oracle's whole Muon step on each
    owned matrix (momentum in float32, weights rounded to their dtype)."""
    for w, g, m in zip(params, grads, moms):
        w_new, m_new, _ = oracle.muon_step_matrix(w.double().numpy(), g.float().numpy(), m.numpy(), lr=lr,
                                                  mu=momentum, nesterov=True, eps=1e-7)
        w.copy_(torch.from_numpy(w_new).to(w.dtype))
        m.copy_(torch.from_numpy(m_new))


SHARD_SHAPES = [(6, 4), (4, 6), (8, 8), (10, 3), (3, 10), (5, 5), (12, 12), (16, 9)]


def _sharded_inputs():
    gen = torch.Generator().manual_seed(0)
    params = [0.02 * torch.randn(r, c, generator=gen) for r, c in SHARD_SHAPES]   # same on every rank
    grads = [torch.randn(r, c, generator=gen) for r, c in SHARD_SHAPES]
    return params, grads


def _sharded_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        params, grads = _sharded_inputs()
        sm = sharded.ShardedMuon(params, device="cpu", step_fn=_oracle_step)
        for _ in range(3):
            sm.step([g if sm.owner[i] == rank else None for i, g in enumerate(grads)], lr=0.02, momentum=0.95)
        out[rank] = ([p.clone() for p in sm.params], sm.owner, sorted(sm.moms),
                     {i: m.clone() for i, m in sm.moms.items()})
    finally:
        dist.destroy_process_group()


def test_sharded_step_gives_every_rank_the_oracles_updated_weights():
    """Two gloo ranks split the matrices by LPT, each runs the oracle's Muon step on its
    own share, and one all-gather gives both ranks every updated weight: the result
    equals the oracle's step on every matrix in one process, bit for bit, and momentum
    lives only on the owning rank."""
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_sharded_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    params, grads = _sharded_inputs()
    moms = [torch.zeros(r, c) for r, c in SHARD_SHAPES]
    for _ in range(3):
        _oracle_step(params, grads, moms, lr=0.02, momentum=0.95)
    owners = set()
    for r in range(world):
        got, owner, mine, mom = out[r]
        for a, b in zip(got, params):
            assert torch.equal(a, b)
        assert mine == [i for i in range(len(SHARD_SHAPES)) if owner[i] == r]  # momentum only where owned
        for i, m in mom.items():
            assert torch.equal(m, moms[i])
        owners |= set(mine)
    assert owners == set(range(len(SHARD_SHAPES))) and len(set(out[0][1])) == 2
