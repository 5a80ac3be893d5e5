"""KV-head tensor parallelism for the CoWA op: which global KV heads (with their query heads) a
rank owns, and the pattern each of its calls passes.

CoWindow Attention picks a head's long-range interval by the head's index in the whole layer
(skillfed.io news summary of 2026-09-30, paragraphs 4 and 6: the pattern follows from positions
and the global KV-head index alone, which keeps the intervals complementary under tensor-parallel
sharding).  A rank that holds the global heads G0 .. G0+n-1 therefore calls the library with
kv_head_base = G0 and h_kv_global = H, and the intervals of all ranks stay complementary.  The op has no exchange step: every rank works on
its own heads; the collectives belong to the projections around it.

Load balance.  A head's interval [b_p, b_p+1) is seen by every later query, so the heads with
early intervals do more work: at N = T = 32768, S = 128, L = 2048, H = D = 8 the visible pairs per
KV head fall from 185.4 M (head 0) to 71.0 M (head 7).  A contiguous split of the heads over P
ranks leaves the rank that holds head 0 with the most work (mean / max = 0.79, 0.72, 0.69 at
P = 2, 4, 8).  Folding the heads instead -- 2P equal blocks of consecutive heads, rank r taking
blocks r and 2P-1-r -- pairs early with late intervals (P = 2: heads {0,1,6,7} and {2,3,4,5};
P = 4: {0,7}, {1,6}, {2,5}, {3,4}; mean / max = 0.998 and 0.994).  A rank then owns at most two
runs of consecutive heads and makes one call per run; the head order is a permutation of the
projection's output columns, fixed when the weights are loaded.  With one KV head per rank
(P = H) no head order balances the work.

Plain host logic; nothing here launches a kernel.
"""

from __future__ import annotations

import dataclasses

import numpy as np

from .cowa import Pattern, visible_counts

ORDERS = ("folded", "contiguous")


@dataclasses.dataclass(frozen=True)
class HeadRun:
    """Consecutive global KV heads G0 .. G0+n-1 of one rank, and their query heads
    G0*grp .. (G0+n)*grp - 1 (query head h reads KV head h // grp)."""

    G0: int
    n: int
    grp: int

    @property
    def q_heads(self) -> range:
        return range(self.G0 * self.grp, (self.G0 + self.n) * self.grp)

    @property
    def kv_heads(self) -> range:
        return range(self.G0, self.G0 + self.n)


def head_owner(G: int, world: int, H: int, order: str = "folded") -> int:
    """The rank that owns global KV head G when H heads are split over `world` ranks.

    contiguous: rank r owns heads r*H/P .. (r+1)*H/P - 1.  folded: the heads form blocks of
    c = H/(2P) consecutive heads (c = 1 when 2P does not divide H) dealt out to ranks 0, 1, ..,
    P-1, then back P-1, .., 0, and so on; with c = H/(2P) that is one pass out and one back."""
    if world < 1 or H % world != 0 or not 0 <= G < H:
        raise ValueError(f"need 0 <= G < H and H % world == 0 (G={G}, H={H}, world={world})")
    if order == "contiguous":
        return G // (H // world)
    if order == "folded":
        c = H // (2 * world) if H % (2 * world) == 0 else 1
        j, r = divmod(G // c, world)
        return r if j % 2 == 0 else world - 1 - r
    raise ValueError(f"order must be one of {ORDERS}")


def kv_head_runs(rank: int, world: int, H: int, grp: int, order: str = "folded") -> list[HeadRun]:
    """The runs of consecutive global KV heads that `rank` owns, in increasing G."""
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside [0, {world})")
    mine = [G for G in range(H) if head_owner(G, world, H, order) == rank]
    runs: list[HeadRun] = []
    for G in mine:
        if runs and runs[-1].G0 + runs[-1].n == G:
            runs[-1] = HeadRun(runs[-1].G0, runs[-1].n + 1, grp)
        else:
            runs.append(HeadRun(G, 1, grp))
    return runs


def run_pattern(pattern: Pattern, run: HeadRun, H: int) -> Pattern:
    """The pattern one call over `run` passes: the layer's windows, the run's first global head as
    kv_head_base and the layer's KV-head count as h_kv_global."""
    return dataclasses.replace(pattern, kv_head_base=run.G0, h_kv_global=H)


def rank_visible_pairs(pattern: Pattern, rank: int, world: int, H: int, grp: int, N: int, B: int = 1,
                       order: str = "folded") -> int:
    """Visible (query, key) pairs of one rank's calls over an N-token prefill, from the library's
    own per-position counts (cowa_visible_counts) of each run."""
    total = 0
    for run in kv_head_runs(rank, world, H, grp, order):
        total += int(visible_counts(run_pattern(pattern, run, H), run.n, N).sum())
    return total * grp * B


def balance(pattern: Pattern, world: int, H: int, grp: int, N: int, B: int = 1, order: str = "folded"):
    """(per-rank visible pairs, mean / max): the fraction of P ideal ranks' throughput that the
    slowest rank allows when time is proportional to visible pairs."""
    per = np.array([rank_visible_pairs(pattern, r, world, H, grp, N, B, order) for r in range(world)],
                   dtype=np.int64)
    return per, float(per.mean() / per.max())
