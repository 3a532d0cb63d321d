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


def test_head_ranges_cover_every_head_once_and_balance():
    from block_sparse_attention_tokens_b200.pipeline import head_range
    for heads in (1, 2, 5, 12, 16, 24, 40):
        for world in range(1, min(heads, 8) + 1):
            ranges = [head_range(r, world, heads) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == heads
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [h1 - h0 for h0, h1 in ranges]
            assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1


def _head_split_main(rank, world, port, out):
    """Each rank evaluates the oracle's attention on its own heads only; the host
    gathers the pieces (test-side reassembly; the library path has no exchange)."""
    import datetime
    import numpy as np
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import oracle as O
    from block_sparse_attention_tokens_b200.pipeline import head_range
    rng = np.random.default_rng(5)                    # the same inputs on every rank
    Bn, H, n, D, blk = 1, 5, 200, 16, 64
    q, k, v = (rng.standard_normal((Bn, n, H, D)) for _ in range(3))
    mask = (rng.random((H, 4, 4)) < 0.6).astype(np.uint8)
    h0, h1 = head_range(rank, world, H)
    o, lse = O.block_sparse_attention(q[:, :, h0:h1], k[:, :, h0:h1], v[:, :, h0:h1],
                                      mask[h0:h1], blk, blk)
    pieces = [None] * world
    dist.all_gather_object(pieces, (h0, h1, o, lse))
    o_all = np.concatenate([p[2] for p in sorted(pieces, key=lambda p: p[0])], axis=2)
    lse_all = np.concatenate([p[3] for p in sorted(pieces, key=lambda p: p[0])], axis=1)
    ref_o, ref_lse = O.block_sparse_attention(q, k, v, mask, blk, blk)
    out[rank] = (bool(np.array_equal(o_all, ref_o)), bool(np.array_equal(lse_all, ref_lse)),
                 (h0, h1))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_split_heads_and_reassemble_exactly():
    world = 2
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_head_split_main, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0][2] == (0, 2) and out[1][2] == (2, 5)
    for rank in range(world):
        assert out[rank][0] and out[rank][1]
