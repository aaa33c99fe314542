"""The multi-GPU bench path's host logic on CPU with gloo, world size 2: the
device times reduce to the slowest rank, and the reported value is the
whole job's FLOPs over that time (attention heads are independent, so ranks
exchange nothing else)."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    local = [100.0 + 50.0 * rank, 10.0 * (rank + 1), 5.0]   # per-rank device ms
    got = bench.reduce_max(local, world, device="cpu")
    out[rank] = got
    dist.barrier()
    dist.destroy_process_group()


def test_reduce_max_and_value_world2():
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert out[0] == out[1] == [150.0, 20.0, 5.0]
    import bench
    # 2 ranks x 10 steps x 1 TFLOP each over the slowest rank's 150 ms
    assert bench.whole_job_tflops(2, 10, 1e12, 150.0) == pytest.approx(20 / 0.150)


def test_flops_counting():
    import bench
    f, b = bench.flops(2, 2048, 12, 64, False)
    assert f == 4 * 2 * 12 * 2048 ** 2 * 64 and b == 2.5 * f
    fc, bc = bench.flops(2, 2048, 12, 64, True)
    assert fc == f / 2 and bc == b / 2


def test_single_rank_is_identity():
    import bench
    assert bench.reduce_max([1.0, 2.0], 1) == [1.0, 2.0]


def test_exp_rate_counts_one_exp_per_unmasked_score():
    import bench
    # 2 x 8 heads x 1024^2 scores, 10 steps in 5 ms on one GPU at 1000 MHz on 100 SMs
    got, peak = bench.exp_rate(2, 1024, 8, False, 5.0, 10, 1, 1000.0, 100)
    assert got == 2 * 8 * 1024 * 1024 * 10 / 5e-3
    assert peak == 16 * 100 * 1000e6
    half, _ = bench.exp_rate(2, 1024, 8, True, 5.0, 10, 1, 1000.0, 100)
    assert half == got / 2
    two, peak2 = bench.exp_rate(2, 1024, 8, False, 5.0, 10, 2, 1000.0, 100)
    assert two == 2 * got and peak2 == 2 * peak
    assert bench.exp_rate(1, 1, 1, False, 1.0, 1, 1, None, 148)[1] is None
