"""Multi-rank timing logic of bench.py on CPU: two gloo ranks, each with its own
batch of work, combine their step times by maximum (weak scaling, no data-path
collective).  Runs without a GPU."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    # rank r pretends its step took 10 + 5 r ms and its attention 8 + r ms
    ms_step, ms_attn = bench.max_over_ranks([10.0 + 5 * rank, 8.0 + rank])
    value = bench.weak_scaling_value(2.0e12, world, ms_step)
    out[rank] = (ms_step, ms_attn, value)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_sum_the_work():
    world = 2
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        ms_step, ms_attn, value = out[rank]
        assert ms_step == 15.0 and ms_attn == 9.0
        # both ranks' 2 TFLOP of work in the slowest rank's 15 ms
        assert abs(value - 2 * 2.0 / 0.015) < 1e-9


def test_single_process_is_the_identity():
    import bench
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    assert abs(bench.weak_scaling_value(1e12, 1, 10.0) - 100.0) < 1e-9
