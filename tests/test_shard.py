"""KV-head tensor parallelism on CPU: which heads a rank owns, that the ranks' calls (patterns with
kv_head_base / h_kv_global) reproduce the whole layer's per-head visibility through the library's
own host arithmetic, that the long-range intervals stay complementary across ranks, the load
balance of the two head orders, and bench.py's per-rank call lists (two gloo ranks, fake compute)."""

import os
import socket
import types

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from oracle import cowa_oracle as orc
from structured_sparse_attention_cowa_b200 import cowa as cw
from structured_sparse_attention_cowa_b200 import shard, synth


@pytest.mark.parametrize("order", shard.ORDERS)
@pytest.mark.parametrize("H,world", [(8, 1), (8, 2), (8, 4), (8, 8), (6, 3), (4, 2), (12, 2)])
def test_every_head_has_exactly_one_owner(order, H, world):
    grp = 3
    owned = sorted(G for r in range(world) for run in shard.kv_head_runs(r, world, H, grp, order) for G in run.kv_heads)
    assert owned == list(range(H))
    for r in range(world):
        runs = shard.kv_head_runs(r, world, H, grp, order)
        assert sum(run.n for run in runs) == H // world
        assert len(runs) <= 2 if order == "folded" else len(runs) == 1
        for run in runs:
            assert list(run.q_heads) == list(range(run.G0 * grp, (run.G0 + run.n) * grp))


def test_folded_order_examples():
    own = lambda P: [[(x.G0, x.n) for x in shard.kv_head_runs(r, P, 8, 5, "folded")] for r in range(P)]
    assert own(2) == [[(0, 2), (6, 2)], [(2, 4)]]
    assert own(4) == [[(0, 1), (7, 1)], [(1, 1), (6, 1)], [(2, 1), (5, 1)], [(3, 2)]]
    assert own(8) == [[(g, 1)] for g in range(8)]
    with pytest.raises(ValueError):
        shard.head_owner(0, 3, 8)


@pytest.mark.parametrize("order", shard.ORDERS)
@pytest.mark.parametrize("world", [1, 2, 4, 8])
def test_rank_patterns_reproduce_the_layer(order, world):
    """Each run's counts (through cowa_visible_counts with the run's kv_head_base) are the layer's
    counts of those heads, and equal the oracle mask's row sums for the same global heads."""
    H, grp, N = 8, 2, 700
    pat = cw.Pattern(24, 50, 640, 8)
    whole = cw.visible_counts(pat, H, N)
    opat = orc.Pattern(S=24, L=50, T=640, D=8)
    for r in range(world):
        for run in shard.kv_head_runs(r, world, H, grp, order):
            rp = shard.run_pattern(pat, run, H)
            assert (rp.kv_head_base, rp.h_kv_global) == (run.G0, H)
            got = cw.visible_counts(rp, run.n, N)
            assert np.array_equal(got, whole[run.G0:run.G0 + run.n])
            for i, G in enumerate(run.kv_heads):
                want = orc.visible_mask(np.arange(N), N, opat, G, H).sum(axis=1)
                assert np.array_equal(got[i], want)


def test_balance_of_the_two_orders():
    """Visible pairs per rank at the 32K training layer (N = T = 32768, S = 128, L = 2048, H_kv = D = 8,
    group 5): the contiguous split leaves the rank with head 0 the most work; folding evens it out."""
    pat = cw.Pattern(128, 2048, 32768, 8)
    whole = bench.visible_pairs(32768, 128, 2048, 32768, 8, 8, 40)
    for P in (1, 2, 4, 8):
        for order in shard.ORDERS:
            per, eff = shard.balance(pat, P, 8, 5, 32768, order=order)
            assert int(per.sum()) == whole
    eff = {(o, P): shard.balance(pat, P, 8, 5, 32768, order=o)[1] for o in shard.ORDERS for P in (2, 4, 8)}
    assert eff[("contiguous", 2)] == pytest.approx(0.7942, abs=1e-4)
    assert eff[("contiguous", 4)] == pytest.approx(0.7195, abs=1e-4)
    assert eff[("folded", 2)] > 0.997 and eff[("folded", 4)] > 0.993
    assert eff[("folded", 8)] == eff[("contiguous", 8)] == pytest.approx(0.6872, abs=1e-4)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _tp_worker(rank, world, port, out):
    """One gloo rank: its own heads' counts through the library, gathered on every rank."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        H, grp, N = 8, 5, 1500
        pat = cw.Pattern(40, 96, 1400, 8)
        mine = {}
        for run in shard.kv_head_runs(rank, world, H, grp, "folded"):
            counts = cw.visible_counts(shard.run_pattern(pat, run, H), run.n, N)
            for i, G in enumerate(run.kv_heads):
                mine[G] = counts[i]
        parts = [None] * world
        dist.all_gather_object(parts, mine)
        out[rank] = parts
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_keep_the_intervals_complementary():
    """With D = H and N <= T the intervals of all ranks partition [S, T): summed over the layer's
    heads, the keys a head sees beyond sink and band are exactly the causal prefix minus sink and
    band (each key in exactly one head's interval)."""
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_tp_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    H, N, S, L, T = 8, 1500, 40, 96, 1400
    pat = cw.Pattern(S, L, T, 8)
    whole = cw.visible_counts(pat, H, N)
    for r in range(world):
        got = {}
        for part in out[r]:
            assert not set(part) & set(got)  # no head computed twice
            got.update(part)
        assert sorted(got) == list(range(H))
        layer = np.stack([got[G] for G in range(H)])
        assert np.array_equal(layer, whole)
        t = np.arange(N)
        sink_band = np.minimum(S, t + 1) + (t + 1 - np.maximum(0, t - L + 1)) - np.maximum(0, np.minimum(S, t + 1) - np.maximum(0, t - L + 1))
        # [S, min(t+1, T)) minus the band (t-L, t]
        lr = np.maximum(0, np.minimum(t + 1, T) - S)
        lr_in_band = np.maximum(0, np.minimum(t + 1, T) - np.maximum(S, t - L + 1))
        assert np.array_equal((layer - sink_band).sum(axis=0), lr - lr_in_band)


class _Recorder:
    """Stands in for the binding's compute calls: records which tensors and pattern each call got."""

    def __init__(self):
        self.calls = []
        self.Pattern = cw.Pattern
        self.lib = cw.lib

    def cowa_fwd(self, q, k, v, pattern, out=None, lse=None, workspace=None):
        self.calls.append(("fwd", q, k, pattern, out, workspace))

    def cowa_bwd(self, q, k, v, o, lse, do, pattern, dq=None, dk=None, dv=None, workspace=None):
        self.calls.append(("bwd", q, k, pattern, dq, workspace))

    def cowa_decode(self, q_t, kc, vc, pos, pattern, out=None, lse=None, workspace=None):
        self.calls.append(("dec", q_t, kc, pattern, out, workspace))

    def workspace_status(self, ws):
        return 0


@pytest.mark.parametrize("order", shard.ORDERS)
@pytest.mark.parametrize("world", [1, 2, 4])
def test_bench_tp_rank_buffers_and_calls(order, world):
    """bench.TpRank on tiny shapes on the CPU: every rank's calls cover its own heads with its own
    buffers and the run's pattern, and the ranks together cover the layer's heads once."""
    c = dict(B=1, N=64, Hq=8, Hkv=4, d=64, S=4, L=8, T=64, D=4)
    dc = dict(B=2, Hq=8, Hkv=4, d=64, T_cap=96, S=4, L=8, T=64, D=4, pos=80)
    seen_q, seen_kv = [], []
    for r in range(world):
        rec = _Recorder()
        tr = bench.TpRank(rec, synth, torch, torch.device("cpu"), r, world, order, c, dc)
        tr.fwd(); tr.bwd(); tr.dec()
        assert tr.launches_per_step == 6 * len(tr.runs)
        assert tr.statuses() == [0] * (3 * len(tr.runs))
        n = len(tr.bufs)
        assert [x[0] for x in rec.calls] == ["fwd"] * n + ["bwd"] * n + ["dec"] * n
        for i, b in enumerate(tr.bufs):
            run = b["run"]
            assert b["q"].shape == (1, 64, 2 * run.n, 64) and b["k"].shape == (1, 64, run.n, 64)
            assert b["kc"].shape == (2, run.n, 96, 64) and b["qt"].shape == (2, 2 * run.n, 64)
            assert b["lse"].shape == (1, 2 * run.n, 64) and b["lsed"].shape == (2, 2 * run.n)
            for kind, j, ws in (("fwd", i, "ws_f"), ("bwd", n + i, "ws_b"), ("dec", 2 * n + i, "ws_d")):
                call = rec.calls[j]
                assert call[5] is b[ws]
                assert call[1] is (b["qt"] if kind == "dec" else b["q"])
                assert call[3].kv_head_base == run.G0 and call[3].h_kv_global == 4
            seen_q += list(run.q_heads)
            seen_kv += list(run.kv_heads)
    assert sorted(seen_q) == list(range(8)) and sorted(seen_kv) == list(range(4))
