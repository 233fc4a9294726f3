"""Multi-rank plumbing of bench.py on CPU: two gloo ranks on 127.0.0.1.

bench.py runs data parallel, one rank per GPU: the masters are the same on
every rank, each rank draws its own batch, every step ends with the sum of dW
over the ranks (the gradient exchange), the ranks meet at a barrier around the
timed region, and the reported time is the slowest rank's.  These tests run
that host logic with world size 2 and no GPU.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        # each rank reports a different per-step time; all must agree on the max
        mx = bench.max_over_ranks(1.5 + rank, world)
        seeds = [bench.replica_seed(rank, r, j) for r in range(bench.ROTATE) for j in range(3)]
        gathered = [None] * world
        dist.all_gather_object(gathered, seeds)
        # the gradient exchange: each rank's dW summed in place
        dw = torch.full((4, 8), float(rank + 1))
        bench.exchange_dw(dw, world)
        out[rank] = (mx, gathered, dw.tolist())
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time_and_draw_distinct_inputs():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 2.5
    seeds0, seeds1 = res[0][1]
    assert len(set(seeds0)) == len(seeds0) and not set(seeds0) & set(seeds1)
    assert res[0][2] == res[1][2] == [[3.0] * 8] * 4  # 1 + 2 on both ranks


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.25, 1) == 3.25
    bench.barrier(1)


def _sum_words_worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from sparse_linear_layers_bitlinear_b200 import sbl

        # words as a shard's sbl_weight_abs_sum writes them: 32-bit pieces,
        # 64-bit bins below 2^60, counts
        g = torch.Generator().manual_seed(100 + rank)
        words = torch.randint(0, 2 ** 60, (sbl.SBL_SUM_WORDS,), generator=g, dtype=torch.int64)
        words[:3] = torch.randint(0, 2 ** 32, (3,), generator=g, dtype=torch.int64)
        mine = words.clone()
        sbl.allreduce_sum_words(words)
        gathered = [None] * world
        dist.all_gather_object(gathered, mine.tolist())
        out[rank] = (words.tolist(), gathered)
    finally:
        dist.destroy_process_group()


def test_row_sharded_scale_words_add_exactly_across_two_gloo_ranks():
    """Step 2 of the row-sharded scale: every rank ends with the word-by-word
    integer sum of all ranks' sum words (no rounding anywhere)."""
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_sum_words_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    expect = [a + b for a, b in zip(*res[0][1])]
    assert res[0][0] == res[1][0] == expect
    assert all(v < 2 ** 63 for v in expect)
