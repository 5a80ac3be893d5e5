"""bench.py's multi-rank plumbing on CPU with two gloo ranks (per-rank seeds differ, the timing
reduction is the max over ranks, the whole-job value uses that max), and its work accounting
(visible pairs of the prefill, visible tokens of a decode step) against the oracle's mask."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from oracle import cowa_oracle as orc


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


@pytest.mark.parametrize("N,S,L,T,D,Hkv,Hq,B,H", [
    (1024, 64, 128, 1024, 4, 4, 8, 1, None),
    (777, 0, 1, 700, 3, 3, 6, 2, None),      # no sink, L = 1, N > T
    (600, 130, 70, 600, 2, 2, 10, 1, None),  # sink not tile aligned, group of 5
    (300, 4, 60, 4, 1, 2, 4, 1, None),       # SWA + sinks (T = S)
    (512, 16, 512, 512, 4, 4, 4, 1, None),   # dense causal
    (400, 8, 40, 400, 4, 2, 4, 1, 4),        # the first 2 of a 4-head layer
])
def test_visible_pairs_match_the_oracle_mask(N, S, L, T, D, Hkv, Hq, B, H):
    """bench.visible_pairs (the FLOP accounting of every bench line) against the oracle's explicit
    mask, summed over positions, KV heads, query heads and batch."""
    pat = orc.Pattern(S=S, L=L, T=T, D=D, h_kv_global=H)
    want = int(orc.visible_counts(N, pat, Hkv).sum()) * (Hq // Hkv) * B
    assert bench.visible_pairs(N, S, L, T, D, Hkv, Hq, B, h_kv_global=H) == want


@pytest.mark.parametrize("pos,S,L,T,D,Hkv", [
    (1023, 64, 128, 1024, 4, 4), (63, 64, 128, 1024, 4, 4), (500, 0, 1, 400, 2, 2), (5000, 16, 100, 2000, 2, 4),
])
def test_decode_visible_tokens_match_the_oracle_mask(pos, S, L, T, D, Hkv):
    pat = orc.Pattern(S=S, L=L, T=T, D=D)
    want = [int(orc.visible_mask(np.array([pos]), pos + 1, pat, g, Hkv).sum()) for g in range(Hkv)]
    assert bench.decode_visible_tokens(pos, S, L, T, D, Hkv) == want


def test_accounting_helpers():
    # the 128K decode configuration: the closed form against the oracle's row count for the first
    # and the last head (the mask of a 131072-wide row is cheap)
    toks = bench.decode_visible_tokens(131071, 128, 4096, 131072, 8, 8)
    pat = orc.Pattern(S=128, L=4096, T=131072, D=8)
    for g in (0, 7):
        assert toks[g] == int(orc.visible_mask(np.array([131071]), 131072, pat, g, 8).sum())
    assert bench.aggregate_tflops(1, 2e12, 1000.0) == pytest.approx(2.0)
