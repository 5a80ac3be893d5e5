"""bench.py's multi-rank plumbing on CPU with two gloo ranks: per-rank seeds differ, the
timing reduction is the max over ranks, and the whole-job value uses that max."""

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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = 10.0 + 5.0 * rank          # the slower rank must win
        worst = bench.max_over_ranks(my_ms, dist, torch.device("cpu"))
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.rank_seed_extra(rank))
        out[rank] = (worst, seeds, bench.aggregate_tflops(world, 1e12, worst))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        worst, seeds, val = out[r]
        assert worst == 15.0
        assert len(set(seeds)) == world
        assert val == pytest.approx(world * 1e12 / 15e-3 / 1e12)


def test_accounting_helpers():
    assert bench.visible_pairs(1024, 64, 128, 1024, 4, 4, 8) == 2119232
    assert bench.decode_visible_tokens(131071, 128, 4096, 131072, 8, 8) == [20592] * 7 + [16496]
    assert bench.aggregate_tflops(1, 2e12, 1000.0) == pytest.approx(2.0)
