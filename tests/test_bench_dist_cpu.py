"""bench.py's multi-rank logic on CPU: 2 gloo ranks (no GPU needed).

Each rank searches its own layer (independent problems, weak scaling); the only
collective is the maximum of the ranks' device times.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from workloads import WORKLOADS


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks([10.0 * rank + 1.0, 5.0 - rank], "cpu")
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
        assert out[0] == [11.0, 5.0] and out[1] == [11.0, 5.0]


def test_single_process_needs_no_collective():
    assert bench.max_over_ranks([3.0, 4.0], "cpu") == [3.0, 4.0]


def test_each_rank_gets_its_own_layer():
    base = WORKLOADS["llama7b_attn_proj_4096x4096x4096"]
    specs = [bench.rank_spec(base, r) for r in range(4)]
    assert len({s.seed for s in specs}) == 4
    assert all((s.M, s.K, s.N) == (base.M, base.K, base.N) for s in specs)


def test_weak_scaling_value():
    # 2 ranks x 10 steps of 1 TFLOP each in 1 s (slowest rank) = 20 TFLOP/s
    assert bench.weak_scaling_tflops(2, 10, 1e12, 1000.0) == pytest.approx(20.0)


def test_reference_arm_runs_on_rank_zero_only():
    args = bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert bench.run_reference(args, rank=1, world=2) == 0
