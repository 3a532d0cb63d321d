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


def test_query_block_ranges_cover_every_block_once_and_balance():
    from block_sparse_attention_tokens_b200.pipeline import qblock_range
    for granule in (1, 2):
        for qblocks in (1, 3, 37, 3544):
            units = -(-qblocks // granule)
            for world in range(1, min(units, 8) + 1):
                ranges = [qblock_range(r, world, qblocks, granule) for r in range(world)]
                assert ranges[0][0] == 0 and ranges[-1][1] == qblocks
                assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
                assert all(b0 % granule == 0 for b0, _ in ranges)     # q-tile aligned
                sizes = [-(-(b1 - b0) // granule) for b0, b1 in ranges]
                assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1


def test_query_block_split_is_chosen_when_heads_do_not_divide():
    # the radial workload (12 heads) over 8 ranks: query blocks; 24 STA heads over 8
    # ranks (tile-ordered anyway): heads
    from block_sparse_attention_tokens_b200 import configs
    w = configs.get("radial_long")
    assert w.heads % 8 != 0 and w.tile is None and w.mask == "radial"
    assert configs.get("sta_720p").heads % 8 == 0


def _qblock_split_main(rank, world, port, out):
    """Each rank evaluates the oracle's attention on its own query blocks of every
    head (all keys); the host gathers the rows (test-side reassembly)."""
    import datetime
    import numpy as np
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import oracle as O
    from block_sparse_attention_tokens_b200.pipeline import qblock_range
    rng = np.random.default_rng(6)                    # the same inputs on every rank
    Bn, H, n, D, blk = 1, 3, 300, 16, 64
    q, k, v = (rng.standard_normal((Bn, n, H, D)) for _ in range(3))
    QB = -(-n // blk)
    mask = (rng.random((1, QB, QB)) < 0.6).astype(np.uint8)
    b0, b1 = qblock_range(rank, world, QB)
    r0, r1 = b0 * blk, min(n, b1 * blk)
    o, lse = O.block_sparse_attention(q[:, r0:r1], k, v, mask[:, b0:b1], blk, blk)
    pieces = [None] * world
    dist.all_gather_object(pieces, (r0, o, lse))
    pieces = sorted(pieces, key=lambda p: p[0])
    o_all = np.concatenate([p[1] for p in pieces], axis=1)
    lse_all = np.concatenate([p[2] for p in pieces], axis=2)
    ref_o, ref_lse = O.block_sparse_attention(q, k, v, mask, blk, blk)
    out[rank] = (bool(np.array_equal(o_all, ref_o)), bool(np.array_equal(lse_all, ref_lse)))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_split_query_blocks_and_reassemble_exactly():
    world = 2
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_qblock_split_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        assert out[rank] == (True, True)
