"""The multi-process (replicas) path of bench.py on CPU: two gloo ranks.

bench.py runs one process per GPU, each serving its own batch with its own copy
of the packed head (no collective on the data path); the only cross-rank step
is the timing, taken as the maximum over ranks, and the reported value is the
whole job's tokens per second.  These tests run that step with the gloo backend.
"""
import importlib.util
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench = _bench()
        ms = bench.max_over_ranks(10.0 + 3.0 * rank, "cpu")   # rank r took 10 + 3r ms
        dist.barrier()
        out[rank] = (ms, bench.job_throughput(world, 64, 100, ms))
    finally:
        dist.destroy_process_group()


def test_single_process_timing_is_its_own():
    bench = _bench()
    assert bench.max_over_ranks(12.5, "cpu") == 12.5
    assert bench.job_throughput(1, 1, 3000, 300.0) == pytest.approx(10000.0)


def test_two_gloo_ranks_take_the_slowest_time():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
        res = dict(out)
    assert sorted(res) == [0, 1]
    for rank in range(world):
        ms, value = res[rank]
        assert ms == 13.0                                   # max over ranks, seen by every rank
        assert value == pytest.approx(2 * 64 * 100 / 0.013)  # both ranks' tokens over the slowest time
