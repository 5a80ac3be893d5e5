"""Plain CPU fp64 oracle for CoWindow Attention (CoWA).

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference legs
may import or call anything in this package.  The library's own call path
(``libcowa.so`` and its Python binding) never touches it, and this module
imports nothing from the library.

What it computes, and where the pages say so
--------------------------------------------
Sources are web pages about CoWA, cited by title and section:

* [NEWS]  "Splitting long-range windows across KV heads beats duplicating them
  at lower cost" (skillfed.io news, 2026-09-30), paragraphs 1-7.
* [ABS]   "CoWindow Attention: Full Causal Coverage Is a Collective Property",
  Abstract (newx.sg paper detail; the same abstract is on the acceptodds.com
  ICLR 2027 submission 1443 page).
* [SWA]   "Sliding Window Attention Beats Linear Attention ...", section
  "Missing Baseline: SWA with Attention Sinks".

The pattern ([NEWS] paragraph 2, [ABS]): every KV head sees a shared
prefix-sink window and a shared near-diagonal window; the rest of the history
is cut into non-overlapping long-range intervals, one per KV head, chosen from
the position and the *global* KV-head index alone ([NEWS] paragraphs 4 and 6).
Each head then runs an ordinary softmax over its own visible keys ([NEWS]
paragraph 7).  CoWA is therefore exact attention under a position-defined
boolean mask, and this oracle is that definition written out: build the mask
explicitly, then dense softmax attention with masked scores at -inf.

Readings of points the pages leave open (each one is this library's choice):

* interval bounds: equal width over ``[S, T)`` with floor boundaries
  ``b_i = S + floor(i*(T-S)/H)``, ``i = 0..H``; ``T`` is a declared span.
* ``D < H`` (the duplicated-window ablation of [NEWS] paragraph 3 at fixed
  per-head widths): global head ``G`` uses slot ``p(G) = (G mod D)*(H/D)``,
  so only ``D`` distinct intervals exist, each repeated over ``H/D`` heads;
  ``D`` must divide ``H``.
* near-diagonal window ``(t-L, t]`` (``L`` keys including ``t``), ``L >= 1``;
  sink ``[0, S)``; GQA map ``g = h // (H_q/H_kv)``; global index
  ``G = kv_head_base + g``; scale ``1/sqrt(d)`` unless given; LSE is the
  natural log of the softmax denominator.

Parity status: every function below is pinned by the CPU tests under
``tests/`` (union = causal prefix, disjoint equal intervals, the dense-causal
and sliding-window special cases checked against library attention routines,
brute-force loops, finite differences, closed-form counts).  The exact
position of the interval boundaries and the D<H slot choice are stated
readings: the pages give no formula, so beyond the invariants they cannot be
checked against the pages (parity for those two choices is unpinned by
construction).
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = [
    "Pattern",
    "interval_bounds",
    "interval_of",
    "visible_mask",
    "visible_counts",
    "attention_fwd",
    "attention_bwd",
    "attention_fwd_rows",
    "attention_bwd_rows",
    "attention_bwd_cols",
    "decode",
    "tile_plan_fwd",
    "tile_plan_bwd",
    "bf16_bits_to_f64",
]


@dataclasses.dataclass(frozen=True)
class Pattern:
    """CoWA window parameters.

    S: prefix-sink size; L: near-diagonal width; T: declared span of the
    long-range region ``[S, T)``; D: number of distinct long-range intervals;
    kv_head_base / h_kv_global: global KV-head indexing ([NEWS] paragraph 6,
    KV-head tensor parallelism); scale: softmax scale (None -> 1/sqrt(d)).
    """

    S: int
    L: int
    T: int
    D: int
    kv_head_base: int = 0
    h_kv_global: int | None = None
    scale: float | None = None

    def H(self, h_kv: int) -> int:
        return self.h_kv_global if self.h_kv_global is not None else h_kv

    def sm_scale(self, d: int) -> float:
        return self.scale if (self.scale is not None and self.scale > 0) else 1.0 / math.sqrt(d)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# Pattern: intervals and the explicit mask ([NEWS] paragraph 2, [ABS])
# ---------------------------------------------------------------------------

def interval_bounds(S: int, T: int, H: int) -> list[int]:
    """Boundaries b_0..b_H of the H equal-width long-range intervals of [S, T)."""
    R = T - S
    return [S + (i * R) // H for i in range(H + 1)]


def interval_of(G: int, pat: Pattern, h_kv: int) -> tuple[int, int]:
    """Long-range interval [lo, hi) of global KV head G (slot (G mod D)*(H/D))."""
    H = pat.H(h_kv)
    b = interval_bounds(pat.S, pat.T, H)
    p = (G % pat.D) * (H // pat.D)
    return b[p], b[p + 1]


def visible_mask(rows: np.ndarray, ncols: int, pat: Pattern, g: int, h_kv: int) -> np.ndarray:
    """Boolean mask M[t, s] = key s visible to query position t for local KV head g.

    visible iff s <= t and (s in sink [0,S) or s in (t-L, t] or s in interval_G).
    """
    t = np.asarray(rows, dtype=np.int64)[:, None]
    s = np.arange(ncols, dtype=np.int64)[None, :]
    lo, hi = interval_of(pat.kv_head_base + g, pat, h_kv)
    causal = s <= t
    sink = s < pat.S
    band = s > t - pat.L
    longr = (s >= lo) & (s < hi)
    return causal & (sink | band | longr)


def visible_counts(N: int, pat: Pattern, h_kv: int) -> np.ndarray:
    """|V_g(t)| for every local KV head g and position t < N, from the explicit mask."""
    out = np.zeros((h_kv, N), dtype=np.int64)
    rows = np.arange(N)
    for g in range(h_kv):
        out[g] = visible_mask(rows, N, pat, g, h_kv).sum(axis=1)
    return out


# ---------------------------------------------------------------------------
# Forward / backward: dense masked softmax attention in fp64
# ---------------------------------------------------------------------------

def _check_shapes(q, k, v):
    B, N, Hq, d = q.shape
    Bk, Nk, Hkv, dk = k.shape
    assert (Bk, Nk, dk) == (B, N, d) and v.shape == k.shape, "q [B,N,Hq,d], k/v [B,N,Hkv,d]"
    assert Hq % Hkv == 0, "H_q must be a multiple of H_kv"
    return B, N, Hq, Hkv, d


def attention_fwd(q: np.ndarray, k: np.ndarray, v: np.ndarray, pat: Pattern):
    """o[B,N,Hq,d] and lse[B,Hq,N] of CoWA attention (self-attention at 0..N-1).

    For head h with g = h // (Hq/Hkv): scores = scale * q_h k_g^T, masked to -inf
    outside V_g(t); lse = log sum exp over each row; o = softmax(scores) v_g.
    """
    q = np.asarray(q, np.float64); k = np.asarray(k, np.float64); v = np.asarray(v, np.float64)
    B, N, Hq, Hkv, d = _check_shapes(q, k, v)
    grp = Hq // Hkv
    scale = pat.sm_scale(d)
    o = np.zeros((B, N, Hq, d))
    lse = np.zeros((B, Hq, N))
    rows = np.arange(N)
    masks = [visible_mask(rows, N, pat, g, Hkv) for g in range(Hkv)]
    for b in range(B):
        for h in range(Hq):
            g = h // grp
            sc = scale * (q[b, :, h, :] @ k[b, :, g, :].T)
            sc = np.where(masks[g], sc, -np.inf)
            m = sc.max(axis=1, keepdims=True)
            e = np.exp(sc - m)
            den = e.sum(axis=1, keepdims=True)
            lse[b, h] = (m + np.log(den))[:, 0]
            o[b, :, h, :] = (e / den) @ v[b, :, g, :]
    return o, lse


def attention_bwd(q, k, v, do, pat: Pattern):
    """Exact gradients (dq, dk, dv) of sum(dO * O) for the forward above.

    With P = softmax of the masked scores: dP = dO v^T, Delta = rowsum(dO * O),
    dS = P * (dP - Delta), dq = scale dS k, dk_g = sum_{h in g} scale dS^T q_h,
    dv_g = sum_{h in g} P^T dO_h.
    """
    q = np.asarray(q, np.float64); k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64); do = np.asarray(do, np.float64)
    B, N, Hq, Hkv, d = _check_shapes(q, k, v)
    grp = Hq // Hkv
    scale = pat.sm_scale(d)
    dq = np.zeros_like(q); dk = np.zeros_like(k); dv = np.zeros_like(v)
    rows = np.arange(N)
    masks = [visible_mask(rows, N, pat, g, Hkv) for g in range(Hkv)]
    for b in range(B):
        for h in range(Hq):
            g = h // grp
            sc = scale * (q[b, :, h, :] @ k[b, :, g, :].T)
            sc = np.where(masks[g], sc, -np.inf)
            m = sc.max(axis=1, keepdims=True)
            e = np.exp(sc - m)
            P = e / e.sum(axis=1, keepdims=True)
            O = P @ v[b, :, g, :]
            dO = do[b, :, h, :]
            dP = dO @ v[b, :, g, :].T
            delta = (dO * O).sum(axis=1, keepdims=True)
            dS = P * (dP - delta)
            dq[b, :, h, :] = scale * (dS @ k[b, :, g, :])
            dk[b, :, g, :] += scale * (dS.T @ q[b, :, h, :])
            dv[b, :, g, :] += P.T @ dO
    return dq, dk, dv


# ---------------------------------------------------------------------------
# Row / column restricted evaluation for long sequences.  Same definition:
# a masked entry contributes exp(-inf) = 0, so evaluating only the rows (or
# the rows that see given columns) changes nothing but the cost.
# ---------------------------------------------------------------------------

def _row_visible_cols(t: int, pat: Pattern, g: int, h_kv: int) -> np.ndarray:
    m = visible_mask(np.array([t]), t + 1, pat, g, h_kv)[0]
    return np.nonzero(m)[0]


def attention_fwd_rows(q, k, v, pat: Pattern, rows, b: int, heads=None, block: int = 256):
    """o[len(rows), len(heads), d] and lse[len(rows), len(heads)] at query positions `rows` of batch b.

    Rows are evaluated in runs of consecutive positions (at most `block` long):
    for each run and KV head the explicit mask is built over [0, t_max], the
    columns that any row of the run sees are gathered once, and each row's
    softmax runs over its own masked scores.  q/k/v may be any array-likes
    indexable as [b, t, h, :] / [b, cols, g, :] that convert to float64.
    """
    Hq = q.shape[2]; Hkv = k.shape[2]; d = q.shape[3]
    grp = Hq // Hkv
    heads = list(range(Hq)) if heads is None else list(heads)
    scale = pat.sm_scale(d)
    rows = np.asarray(rows, dtype=np.int64)
    o = np.zeros((len(rows), len(heads), d))
    lse = np.zeros((len(rows), len(heads)))
    order = np.argsort(rows, kind="stable")
    srt = rows[order]
    # runs of consecutive sorted positions
    starts = [0] + [i for i in range(1, len(srt)) if srt[i] != srt[i - 1] + 1 or i % block == 0]
    bounds = list(zip(starts, starts[1:] + [len(srt)]))
    by_g = {}
    for hi_, h in enumerate(heads):
        by_g.setdefault(h // grp, []).append((hi_, h))
    for a0, a1 in bounds:
        run = srt[a0:a1]
        idx = order[a0:a1]
        tmax = int(run[-1])
        for g, hs in by_g.items():
            m = visible_mask(run, tmax + 1, pat, g, Hkv)
            cols = np.nonzero(m.any(axis=0))[0]
            mm = m[:, cols]
            kk = np.asarray(k[b, cols, g, :], np.float64)
            vv = np.asarray(v[b, cols, g, :], np.float64)
            for hi_, h in hs:
                qh = np.asarray(q[b, run, h, :], np.float64)
                sc = np.where(mm, scale * (qh @ kk.T), -np.inf)
                mx = sc.max(axis=1, keepdims=True)
                e = np.exp(sc - mx)
                den = e.sum(axis=1, keepdims=True)
                lse[idx, hi_] = (mx + np.log(den))[:, 0]
                o[idx, hi_] = (e / den) @ vv
    return o, lse


def _block_visible(run, pat, g, Hkv):
    """Mask rows `run` x the columns any of them sees, and those column indices."""
    tmax = int(run[-1])
    m = visible_mask(run, tmax + 1, pat, g, Hkv)
    cols = np.nonzero(m.any(axis=0))[0]
    return m[:, cols], cols


def attention_bwd_rows(q, k, v, do, pat: Pattern, rows, b: int, heads=None, block: int = 256):
    """dq[len(rows), len(heads), d] at query positions `rows` of batch b (row-local).

    For each row: P over its visible keys, O = P v, Delta = dO.O, dS = P (dO v^T - Delta),
    dq = scale dS k.  Consecutive rows are evaluated together as in attention_fwd_rows.
    """
    Hq = q.shape[2]; Hkv = k.shape[2]; d = q.shape[3]
    grp = Hq // Hkv
    heads = list(range(Hq)) if heads is None else list(heads)
    scale = pat.sm_scale(d)
    rows = np.asarray(rows, dtype=np.int64)
    dq = np.zeros((len(rows), len(heads), d))
    order = np.argsort(rows, kind="stable")
    srt = rows[order]
    starts = [0] + [i for i in range(1, len(srt)) if srt[i] != srt[i - 1] + 1 or i % block == 0]
    by_g = {}
    for hi_, h in enumerate(heads):
        by_g.setdefault(h // grp, []).append((hi_, h))
    for a0, a1 in zip(starts, starts[1:] + [len(srt)]):
        run = srt[a0:a1]
        idx = order[a0:a1]
        for g, hs in by_g.items():
            mm, cols = _block_visible(run, pat, g, Hkv)
            kk = np.asarray(k[b, cols, g, :], np.float64)
            vv = np.asarray(v[b, cols, g, :], np.float64)
            for hi_, h in hs:
                qh = np.asarray(q[b, run, h, :], np.float64)
                doh = np.asarray(do[b, run, h, :], np.float64)
                sc = np.where(mm, scale * (qh @ kk.T), -np.inf)
                e = np.exp(sc - sc.max(axis=1, keepdims=True))
                P = e / e.sum(axis=1, keepdims=True)
                O = P @ vv
                delta = (doh * O).sum(axis=1, keepdims=True)
                dS = P * (doh @ vv.T - delta)
                dq[idx, hi_] = scale * (dS @ kk)
    return dq


def attention_bwd_cols(q, k, v, do, pat: Pattern, b: int, g: int, cols, row_block: int = 512):
    """dk_g[cols], dv_g[cols] (local KV head g, batch b) from every row that sees those columns.

    Rows that see column s are found from the explicit mask; their softmax
    statistics (lse, Delta = rowsum(dO*O)) are recomputed here from scratch over
    each row's own visible keys.
    """
    Hq = q.shape[2]; Hkv = k.shape[2]; d = q.shape[3]; N = q.shape[1]
    grp = Hq // Hkv
    scale = pat.sm_scale(d)
    cols = np.asarray(cols, dtype=np.int64)
    dk = np.zeros((len(cols), d)); dv = np.zeros((len(cols), d))
    kc = np.asarray(k[b, cols, g, :], np.float64); vc = np.asarray(v[b, cols, g, :], np.float64)
    # rows that see at least one requested column
    seen_rows = np.zeros(N, bool)
    for s in cols:
        t = np.arange(s, N)
        seen_rows[t[visible_mask(t, s + 1, pat, g, Hkv)[:, s]]] = True
    rows_all = np.nonzero(seen_rows)[0]
    for r0 in range(0, len(rows_all), row_block):
        run = rows_all[r0:r0 + row_block]
        mm, vcols = _block_visible(run, pat, g, Hkv)
        kk = np.asarray(k[b, vcols, g, :], np.float64)
        vv = np.asarray(v[b, vcols, g, :], np.float64)
        seen = visible_mask(run, N, pat, g, Hkv)[:, cols]
        for h in range(g * grp, (g + 1) * grp):
            qh = np.asarray(q[b, run, h, :], np.float64)
            doh = np.asarray(do[b, run, h, :], np.float64)
            sc = np.where(mm, scale * (qh @ kk.T), -np.inf)
            m = sc.max(axis=1, keepdims=True)
            e = np.exp(sc - m)
            den = e.sum(axis=1, keepdims=True)
            O = (e / den) @ vv
            delta = (doh * O).sum(axis=1, keepdims=True)
            # P at the requested columns: exp(score - lse) where visible, else 0
            Pc = np.where(seen, np.exp(scale * (qh @ kc.T) - (m + np.log(den))), 0.0)
            dSc = Pc * (doh @ vc.T - delta)
            dv += Pc.T @ doh
            dk += scale * (dSc.T @ qh)
    return dk, dv


# ---------------------------------------------------------------------------
# Decode: the row t = pos of the same definition over a KV cache
# ---------------------------------------------------------------------------

def decode(q_t, k_cache, v_cache, pos, pat: Pattern):
    """o[B,Hq,d], lse[B,Hq] for one new token per sequence at position pos[b].

    q_t [B,Hq,d]; caches [B,Hkv,T_cap,d] holding keys/values at 0..pos[b]
    (the new token's own K/V already written at pos[b]).
    """
    B, Hq, d = q_t.shape
    Hkv = k_cache.shape[1]
    grp = Hq // Hkv
    scale = pat.sm_scale(d)
    o = np.zeros((B, Hq, d)); lse = np.zeros((B, Hq))
    for b in range(B):
        t = int(pos[b])
        for g in range(Hkv):
            cols = _row_visible_cols(t, pat, g, Hkv)
            kk = np.asarray(k_cache[b, g, cols, :], np.float64)
            vv = np.asarray(v_cache[b, g, cols, :], np.float64)
            for h in range(g * grp, (g + 1) * grp):
                sc = scale * (kk @ np.asarray(q_t[b, h], np.float64))
                m = sc.max(); e = np.exp(sc - m); den = e.sum()
                lse[b, h] = m + math.log(den)
                o[b, h] = (e / den) @ vv
    return o, lse


# ---------------------------------------------------------------------------
# Tile plans, read off the explicit mask
# ---------------------------------------------------------------------------

def tile_plan_fwd(N: int, BM: int, BN: int, pat: Pattern, h_kv: int):
    """For each (q-tile i, local KV head g): sorted list of (kv-tile j, full).

    Tile (i, j) is visited iff any element of its block of the mask is set, and
    is full iff every element over the valid rows (< N) and columns (< N) is set.
    """
    nq = -(-N // BM); nk = -(-N // BN)
    rows = np.arange(N)
    plan = {}
    for g in range(h_kv):
        M = visible_mask(rows, N, pat, g, h_kv)
        for i in range(nq):
            blk_r = M[i * BM: min(N, (i + 1) * BM)]
            lst = []
            for j in range(nk):
                blk = blk_r[:, j * BN: min(N, (j + 1) * BN)]
                if blk.any():
                    lst.append((j, bool(blk.all())))
            plan[(i, g)] = lst
    return plan


def tile_plan_bwd(N: int, BM: int, BN: int, pat: Pattern, h_kv: int):
    """For each (kv-tile j, local KV head g): sorted list of q-tiles i whose block is non-empty."""
    nq = -(-N // BM); nk = -(-N // BN)
    rows = np.arange(N)
    plan = {}
    for g in range(h_kv):
        M = visible_mask(rows, N, pat, g, h_kv)
        for j in range(nk):
            col = M[:, j * BN: min(N, (j + 1) * BN)]
            plan[(j, g)] = [i for i in range(nq) if col[i * BM: min(N, (i + 1) * BM)].any()]
    return plan
