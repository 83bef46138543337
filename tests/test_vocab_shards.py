"""Vocabulary-sharded head: host-side split and exchange (CPU).

A sharded head gives each GPU a contiguous range of vocabulary rows (whole
128-row tiles, R and B replicated); the only cross-GPU step is an all-gather of
per-token partial softmax statistics in rank order.  The GPU side (partials and
their merge) is checked in test_gpu_parity.py.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import archead_inputs as gen


@pytest.fixture(scope="module")
def qoh():
    import quantized_output_head_b200 as m
    return m


@pytest.mark.parametrize("V,world", [(1000, 3), (151936, 8), (300, 4), (128, 2), (129, 2)])
def test_shard_rows_cover_the_vocabulary_in_tiles(qoh, V, world):
    ranges = [qoh.shard_rows(V, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == V
    for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
        assert a1 == b0                                   # contiguous, no overlap, rank order
    for v0, v1 in ranges:
        assert v0 % 128 == 0 and (v1 % 128 == 0 or v1 == V)
    sizes = [-(-(v1 - v0) // 128) for v0, v1 in ranges]
    assert max(sizes) - min(sizes) <= 1                   # balanced in whole tiles


def test_shard_components_slice_rows_and_share_the_rest(qoh):
    shape = gen.HeadShape(1000, 256, 32, 8, 64, 64)
    comps = gen.random_components(shape, seed=11)
    part = qoh.shard_components(comps, 384, 768)
    for k in ("L", "s_L", "q", "s_res", "A", "s_A"):
        assert np.array_equal(part[k], comps[k][384:768])
    for k in ("R", "s_R", "B", "s_B"):
        assert part[k] is comps[k]


def test_shard_abi_argument_checks(qoh):
    L = qoh._lib
    assert L.archead_set_vocab_shard(None, 0, 10) == qoh.ARCHEAD_EINVAL
    assert L.archead_shard_partials(None, 4096, 1, None, 4096, 4096, 1 << 20, None) == qoh.ARCHEAD_EINVAL
    assert L.archead_merge_shards(None, 2, 4, 4096, None, None, None) == qoh.ARCHEAD_EINVAL
    assert L.archead_merge_shards(4096, 0, 4, 4096, None, None, None) == qoh.ARCHEAD_EINVAL
    assert L.archead_merge_shards(4096 + 4, 2, 4, 4096, None, None, None) == qoh.ARCHEAD_EALIGN


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import quantized_output_head_b200 as qoh
        T = 5
        mine = torch.full((T, 4), float(rank)) + torch.arange(T, dtype=torch.float32)[:, None]
        # sampling pairs: (perturbed value, global row as int32 bits)
        pairs = torch.stack([torch.full((T,), 10.0 * rank),
                             torch.arange(T, dtype=torch.int32).add(100 * rank).view(torch.float32)], dim=1)
        out[rank] = (qoh.gather_partials(mine).numpy(), qoh.gather_partials(pairs).numpy())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_gather_partials_in_rank_order():
    """Both kinds of shard partials (softmax statistics, sampling pairs) cross
    the ranks bit for bit and in rank order."""
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
        res = dict(out)
    for rank in range(world):
        g, pr = res[rank]
        assert g.shape == (world, 5, 4) and pr.shape == (world, 5, 2)
        for r in range(world):
            assert np.array_equal(g[r], np.full((5, 4), float(r)) + np.arange(5)[:, None])
            assert np.array_equal(pr[r, :, 0], np.full(5, 10.0 * r))
            assert np.array_equal(pr[r, :, 1].view(np.int32), np.arange(5) + 100 * r)
