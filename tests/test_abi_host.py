"""Host-side checks of libcowa.so: it loads, exports every function include/cowa.h declares,
its planner matches the oracle's mask-derived plan bit for bit, and bad arguments return
the documented status before any launch.  No GPU is touched here."""

import ctypes
import os
import re

import numpy as np
import pytest

from oracle import cowa_oracle as orc
from structured_sparse_attention_cowa_b200 import cowa as cw

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    txt = open(os.path.join(ROOT, "include", "cowa.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(cowa_[a-z_0-9]+)\s*\(", txt)))


def test_library_exports_every_declared_symbol():
    L = cw.lib()
    names = _declared_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(L, n), n
    assert L.cowa_version() >= 1


def test_debug_library_builds_and_exports_every_declared_symbol():
    """The self-checking build (COWA_DEBUG=1, libcowa_debug.so) is the same ABI."""
    from structured_sparse_attention_cowa_b200 import build as cbuild

    L = ctypes.CDLL(cbuild.build(debug=True))
    for n in _declared_functions():
        assert hasattr(L, n), n
    assert L.cowa_status_string(7) != 0


def _oracle_pattern(p: cw.Pattern):
    return orc.Pattern(S=p.S, L=p.L, T=p.T, D=p.D, kv_head_base=p.kv_head_base,
                       h_kv_global=p.h_kv_global or None)


PLAN_CASES = [
    # N, Hkv, BM, BN, pattern
    (1024, 4, 128, 128, cw.Pattern(64, 128, 1024, 4)),       # tiny config
    (700, 2, 128, 128, cw.Pattern(16, 2**31 - 1, 700, 2)),   # window of INT_MAX (dense causal): no overflow
    (700, 4, 128, 128, cw.Pattern(16, 50, 2**31 - 1, 4)),    # declared span of INT_MAX: intervals past N
    (700, 2, 128, 128, cw.Pattern(2**31 - 1, 1, 2**31 - 1, 2)),  # sink of INT_MAX: every key a sink key
    (1024, 4, 128, 128, cw.Pattern(64, 128, 1024, 2)),       # duplicated D=2
    (1024, 4, 128, 128, cw.Pattern(64, 128, 1024, 1)),       # duplicated D=1
    (1000, 4, 128, 128, cw.Pattern(64, 128, 1000, 4)),       # ragged tail
    (777, 3, 64, 32, cw.Pattern(0, 1, 700, 3)),              # no sink, L=1, N > T
    (600, 2, 128, 128, cw.Pattern(130, 70, 600, 2)),         # sink not tile aligned
    (512, 4, 128, 128, cw.Pattern(16, 512, 512, 4)),         # dense causal (L >= T)
    (300, 4, 32, 32, cw.Pattern(4, 60, 4, 1)),               # SWA + sinks (T = S)
    (257, 2, 128, 128, cw.Pattern(3, 9, 257, 2, kv_head_base=2, h_kv_global=4)),  # TP rank
]


@pytest.mark.parametrize("N,Hkv,BM,BN,pat", PLAN_CASES)
def test_host_plans_match_mask_bit_exact(N, Hkv, BM, BN, pat):
    op = _oracle_pattern(pat)
    fwd = cw.plan_debug(pat, Hkv, N, BM, BN, 0)
    want = sorted((g, i, j, int(full)) for (i, g), lst in orc.tile_plan_fwd(N, BM, BN, op, Hkv).items()
                  for j, full in lst)
    assert sorted(map(tuple, fwd.tolist())) == want
    bwd = cw.plan_debug(pat, Hkv, N, BM, BN, 1)
    want_b = sorted((g, j, i, 0) for (j, g), lst in orc.tile_plan_bwd(N, BM, BN, op, Hkv).items() for i in lst)
    assert sorted(map(tuple, bwd.tolist())) == want_b


@pytest.mark.parametrize("N,Hkv,BM,BN,pat", PLAN_CASES)
def test_visible_counts_bit_exact(N, Hkv, BM, BN, pat):
    got = cw.visible_counts(pat, Hkv, N)
    want = orc.visible_counts(N, _oracle_pattern(pat), Hkv)
    assert np.array_equal(got, want)


def _random_plan_cases(n, seed):
    """Seeded random configurations across the planner's edge classes: T - S not divisible by H,
    S = 0, S >= T (no intervals), L = 1, L >= T (dense causal), N < T and N > T, tile sizes
    32 / 64 / 128, duplicated windows (D < H) and a KV-head offset (tensor-parallel rank)."""
    rng = np.random.default_rng(seed)
    cases = []
    for _ in range(n):
        H = int(rng.choice([1, 2, 3, 4, 6, 8]))
        D = int(rng.choice([x for x in range(1, H + 1) if H % x == 0]))
        N = int(rng.integers(1, 520))
        T = int(rng.integers(1, 640))
        S = int(rng.choice([0, int(rng.integers(0, T + 1)), T]))
        L = int(rng.choice([1, int(rng.integers(1, 200)), T + 5]))
        BM, BN = int(rng.choice([32, 64, 128])), int(rng.choice([32, 64, 128]))
        P = int(rng.choice([1, 2])) if H % 2 == 0 else 1  # ranks sharing the H KV heads
        Hkv = H // P
        base = int(rng.integers(0, P)) * Hkv
        pat = cw.Pattern(S, L, T, D, kv_head_base=base, h_kv_global=H if P > 1 else 0)
        cases.append((N, Hkv, BM, BN, pat))
    return cases


@pytest.mark.parametrize("N,Hkv,BM,BN,pat", _random_plan_cases(40, seed=2027))
def test_random_plans_and_counts_match_the_mask(N, Hkv, BM, BN, pat):
    """Host forward / backward tile plans and visible counts against the oracle's explicit mask,
    bit-exact, over random configurations."""
    test_host_plans_match_mask_bit_exact(N, Hkv, BM, BN, pat)
    test_visible_counts_bit_exact(N, Hkv, BM, BN, pat)


def _closed_form_counts(N, S, L, T, H, D, g):
    """|sink U band U interval| per position by inclusion-exclusion (vectorised over t)."""
    b = [S + (i * (T - S)) // H for i in range(H + 1)]
    p = (g % D) * (H // D)
    lo, hi = b[p], b[p + 1]
    t = np.arange(N, dtype=np.int64)
    def inter(a0, a1, b0, b1):
        return np.maximum(0, np.minimum(a1, b1) - np.maximum(a0, b0))
    A = (np.zeros_like(t), np.minimum(S, t + 1))
    Bd = (np.maximum(0, t - L + 1), t + 1)
    C = (np.full_like(t, lo), np.minimum(hi, t + 1))
    n = lambda r: np.maximum(0, r[1] - r[0])
    ab = inter(*A, *Bd); ac = inter(*A, *C); bc = inter(*Bd, *C)
    abc = np.maximum(0, np.minimum(np.minimum(A[1], Bd[1]), C[1]) - np.maximum(np.maximum(A[0], Bd[0]), C[0]))
    return n(A) + n(Bd) + n(C) - ab - ac - bc + abc


@pytest.mark.parametrize("N,S,L,T,H,D", [(32768, 128, 2048, 32768, 8, 8), (131072, 128, 4096, 131072, 8, 8),
                                          (8192, 128, 1024, 8192, 8, 2)])
def test_visible_counts_of_the_long_configs(N, S, L, T, H, D):
    """Host planner counts at the 8K / 32K / 128K shapes against a closed form, and the union
    over heads covers the causal prefix."""
    pat = cw.Pattern(S, L, T, D)
    c = cw.visible_counts(pat, H, N)
    for g in range(H):
        assert np.array_equal(c[g], _closed_form_counts(N, S, L, T, H, D, g))
    if D == H:
        assert (c.sum(0) >= np.arange(1, N + 1)).all()


# ---------------------------------------------------------------------------- validation
def _t(ptr=0x10000, sb=1 << 20, st=1024, sh=128):
    return cw.c_tensor(ptr, sb, st, sh)


def _fwd(pat, B=1, N=128, Hq=8, Hkv=4, d=128, q=None, lse=0x20000, ws=0x40000, ws_bytes=1 << 20):
    p = pat.c() if pat is not None else None
    return cw.lib().cowa_fwd(ctypes.byref(p) if p is not None else None, B, N, Hq, Hkv, d, q or _t(), _t(), _t(),
                             _t(), lse, ws, ws_bytes, None)


@pytest.mark.parametrize("kwargs,status", [
    (dict(pat=None), 1),
    (dict(pat=cw.Pattern(64, 0, 1024, 4)), 1),          # L = 0
    (dict(pat=cw.Pattern(64, 8, 32, 4)), 1),            # T < S
    (dict(pat=cw.Pattern(64, 8, 1024, 3)), 1),          # D does not divide H
    (dict(pat=cw.Pattern(64, 8, 1024, 4), Hq=6), 1),    # Hq % Hkv
    (dict(pat=cw.Pattern(64, 8, 1024, 4), d=96), 2),    # head dim
    (dict(pat=cw.Pattern(64, 8, 1024, 4), Hq=40, Hkv=4), 2),  # group of 10 > 8
    (dict(pat=cw.Pattern(64, 8, 1024, 4), q=cw.c_tensor(0x10008, 1 << 20, 1024, 128)), 3),  # misaligned ptr
    (dict(pat=cw.Pattern(64, 8, 1024, 4), q=cw.c_tensor(0x10000, 1 << 20, 1020, 128)), 3),  # misaligned stride
    (dict(pat=cw.Pattern(64, 8, 1024, 4), q=cw.c_tensor(0, 1 << 20, 1024, 128)), 1),        # null
    (dict(pat=cw.Pattern(64, 8, 1024, 4), lse=0), 1),
    (dict(pat=cw.Pattern(64, 8, 1024, 4), ws_bytes=16), 4),
    (dict(pat=cw.Pattern(64, 8, 1024, 4), ws=0x40010), 4),  # workspace not 256-aligned
    (dict(pat=cw.Pattern(64, 8, 1024, 4, kv_head_base=2, h_kv_global=4)), 1),  # base + Hkv > H
    (dict(pat=cw.Pattern(64, 8, 1024, 4, kv_head_base=2**31 - 2, h_kv_global=4)), 1),  # base + Hkv wraps
])
def test_fwd_rejects_bad_arguments_before_launch(kwargs, status):
    assert _fwd(**kwargs) == status


@pytest.mark.parametrize("Nq,Nk,off,status", [
    (128, 128, 1, 1),     # the block's last query position is past the keys
    (100, 300, 201, 1),
    (64, 64, -1, 1),      # negative offset
    (64, 0, 0, 1),        # no keys
    (0, 64, 0, 1),        # no queries
])
def test_fwd_chunk_rejects_bad_offsets_before_launch(Nq, Nk, off, status):
    p = cw.Pattern(64, 8, 1024, 4).c()
    assert cw.lib().cowa_fwd_chunk(ctypes.byref(p), 1, Nq, Nk, off, 8, 4, 128, _t(), _t(), _t(), _t(), 0x20000,
                                   0x40000, 1 << 20, None) == status


@pytest.mark.parametrize("pat,Hkv", [
    (cw.Pattern(128, 4096, 131072, 8), 8),
    (cw.Pattern(20, 100, 2000, 2), 2),
    (cw.Pattern(0, 70, 1800, 4), 4),
    (cw.Pattern(64, 256, 1500, 1), 2),
    (cw.Pattern(16, 90, 16, 2), 2),
    (cw.Pattern(3, 9, 257, 2, kv_head_base=2, h_kv_global=4), 2),
])
def test_compact_cache_rows_hold_every_visible_position(pat, Hkv):
    """The compacted layout has room for what decode can see at any position: the sink, the
    band rounded out to 64-aligned blocks, and each head's interval from its 64-aligned start;
    at 128K it is 20,736 rows per head (6.3x fewer than the 131,072 of the full cache)."""
    rows = cw.lib().cowa_compact_rows(ctypes.byref(pat.c()), Hkv)
    H = pat.h_kv_global or Hkv
    b = orc.interval_bounds(pat.S, pat.T, H)
    up = lambda x: -(-x // 64) * 64
    slots = range(0, H, H // pat.D)  # the D distinct interval slots (G mod D) * (H / D)
    need_iv = max([b[j + 1] - b[j] // 64 * 64 for j in slots if b[j + 1] > b[j]], default=0)
    # every 64-aligned block of the band (at most L + 63 positions back from t) fits the ring
    assert rows >= up(pat.S) + up(pat.L + 63) + up(need_iv)
    assert rows <= up(pat.S) + up(pat.L) + 64 + up(need_iv)
    if (pat.S, pat.L, pat.T, pat.D) == (128, 4096, 131072, 8):
        assert rows == 20736


@pytest.mark.parametrize("pat,Hkv", [
    (cw.Pattern(20, 100, 2000, 2), 2),
    (cw.Pattern(0, 70, 1800, 4), 4),
    (cw.Pattern(64, 256, 1500, 1), 2),
    (cw.Pattern(16, 90, 16, 2), 2),
    (cw.Pattern(3, 9, 257, 2, kv_head_base=2, h_kv_global=4), 2),
])
def test_compact_layout_holds_every_visible_key_at_every_position(pat, Hkv):
    """Replays appends position by position on the documented layout (sink row p, ring row
    S64 + p mod R, interval row S64 + R + p - round_down64(lo)), reading the row count from the
    library, and checks that at every decode position every key the oracle's mask makes visible
    is still in its region, read as whole 64-aligned blocks that stay inside that region."""
    rows = cw.lib().cowa_compact_rows(ctypes.byref(pat.c()), Hkv)
    H = pat.h_kv_global or Hkv
    S64 = -(-pat.S // 64) * 64
    R = -(-pat.L // 64) * 64 + 64
    b = orc.interval_bounds(pat.S, pat.T, H)
    N = 700
    op = _oracle_pattern(pat)
    for g in range(Hkv):
        mask_g = orc.visible_mask(np.arange(N), N, op, g, Hkv)  # [N, N]
        G = pat.kv_head_base + g
        slot = (G % pat.D) * (H // pat.D)
        lo, hi = b[slot], b[slot + 1]
        lo64 = lo // 64 * 64
        store = {}  # row -> position held
        for t in range(N):
            store[S64 + t % R] = t                      # append position t
            if t < pat.S:
                store[t] = t
            if lo <= t < hi:
                store[S64 + R + t - lo64] = t
            for s_ in np.nonzero(mask_g[t])[0]:
                if s_ < pat.S:
                    row, blk = s_, (s_ // 64 * 64, s_ // 64 * 64 + 64, 0, S64)
                elif s_ > t - pat.L:
                    row = S64 + s_ % R
                    p0 = s_ // 64 * 64
                    blk = (S64 + p0 % R, S64 + p0 % R + 64, S64, S64 + R)
                else:
                    assert lo <= s_ < hi
                    row = S64 + R + s_ - lo64
                    blk = (S64 + R + (s_ // 64 * 64 - lo64), S64 + R + (s_ // 64 * 64 - lo64) + 64, S64 + R, rows)
                assert store.get(row) == s_, (g, t, s_)
                assert blk[2] <= blk[0] and blk[1] <= blk[3], (g, t, s_, blk)


def test_bwd_workspace_holds_the_split_of_long_key_tiles():
    """The backward splits long dK/dV key tiles only when a call has few KV heads: the 8-head 32K
    layer needs only the row statistics, one of its KV heads alone (a rank of KV-head tensor
    parallelism) also the chunk table and fp32 partials."""
    L = cw.lib()

    def ws(pat, B, N, Hq, Hkv):
        return L.cowa_bwd_workspace_size(ctypes.byref(pat.c()), B, N, Hq, Hkv, 128)

    stats = 256 + 2 * 40 * 32768 * 4
    assert ws(cw.Pattern(128, 2048, 32768, 8), 1, 32768, 40, 8) == stats
    one = ws(cw.Pattern(128, 2048, 32768, 8, kv_head_base=0, h_kv_global=8), 1, 32768, 5, 1)
    # head 0: the sink tile and the 32 tiles of its interval, in chunks of 78 query tiles
    assert one == 256 + 2 * 5 * 32768 * 4 + (121 * 16 + 255) // 256 * 256 + 121 * 2 * 128 * 128 * 4
    last = ws(cw.Pattern(128, 2048, 32768, 8, kv_head_base=7, h_kv_global=8), 1, 32768, 5, 1)
    assert last == 256 + 2 * 5 * 32768 * 4 + 256 + 13 * 2 * 128 * 128 * 4


def _split_plan_bytes(S, L, T, D, H, G0, B, N, Hq, Hkv, d):
    """The key-tile split rule restated from its description: a key tile's query range is every
    query tile from its own to the end if its keys include sink or interval keys, else up to the
    end of the band; chunks of (sum of ranges x B / 148) query tiles, at least 8, when the longest
    range exceeds that; per chunk a 16-byte table entry and fp32 partial dV, dK."""
    nq = (N + 127) // 128

    def bound(i):
        return S + (i * (T - S)) // H

    total, ranges = 0, []
    for g in range(Hkv):
        slot = ((G0 + g) % D) * (H // D)
        lo, hi = bound(slot), bound(slot + 1)
        for j in range(nq):
            s0, s1 = j * 128, min(N, j * 128 + 128)
            special = s0 < S or (lo < hi and lo < s1 and hi > s0)
            end = N if special else min(N, s1 - 1 + L)
            n = (max(s0, end) + 127) // 128 - s0 // 128
            ranges.append(n)
            total += n
    chunk = max(8, total * B // 148)
    if max(ranges) <= chunk:
        return 0
    entries = B * sum((n + chunk - 1) // chunk for n in ranges if n > chunk)
    return (entries * 16 + 255) // 256 * 256 + entries * 2 * 128 * d * 4


def test_bwd_workspace_matches_the_split_rule_on_random_shapes():
    L = cw.lib()
    rng = np.random.default_rng(5)
    for _ in range(60):
        H = int(rng.choice([1, 2, 4, 8]))
        D = int(rng.choice([x for x in (1, 2, 4, 8) if H % x == 0]))
        Hkv = int(rng.integers(1, H + 1))
        G0 = int(rng.integers(0, H - Hkv + 1))
        grp = int(rng.choice([1, 2, 5, 8]))
        B, d = int(rng.integers(1, 3)), int(rng.choice([64, 128]))
        N = int(rng.integers(1, 6000))
        S = int(rng.integers(0, 300))
        T = S + int(rng.integers(0, 7000))
        Lw = int(rng.choice([1, 64, 257, 2048, 2**31 - 1]))
        pat = cw.Pattern(S, Lw, T, D, kv_head_base=G0, h_kv_global=H)
        got = L.cowa_bwd_workspace_size(ctypes.byref(pat.c()), B, N, grp * Hkv, Hkv, d)
        n_pad = (N + 127) // 128 * 128
        want = 256 + (2 * B * grp * Hkv * n_pad * 4 + 255) // 256 * 256 + \
            _split_plan_bytes(S, Lw, T, D, H, G0, B, N, grp * Hkv, Hkv, d)
        assert got == want, (S, Lw, T, D, H, G0, B, N, grp, Hkv, d, got, want)


def test_bwd_varlen_workspace_reserves_the_split_only_when_it_can_happen():
    """A packed batch plans its key-tile split on the device, so its workspace reserves room as
    for one sequence of all its rows: nothing for the 8-head 32K layer, table slots (twice that
    plan's 121 chunks + 64), tile flags and partials for one KV head of it."""
    L = cw.lib()

    def ws(pat, n_seq, total, Hq, Hkv):
        return L.cowa_bwd_varlen_workspace_size(ctypes.byref(pat.c()), n_seq, total, Hq, Hkv, 128)

    n_seq, total = 3, 32768
    rows = (total // 128 + n_seq) * 128
    seq_tab = (3 * n_seq + 1) * 4
    base = lambda Hq: 256 + (seq_tab + 255) // 256 * 256 + 2 * Hq * rows * 4
    assert ws(cw.Pattern(128, 2048, 32768, 8), n_seq, total, 40, 8) == base(40)
    cap = 2 * 121 + 64
    flags = (1 * (rows // 128) * 4 + 255) // 256 * 256
    one = ws(cw.Pattern(128, 2048, 32768, 8, kv_head_base=0, h_kv_global=8), n_seq, total, 5, 1)
    assert one == base(5) + flags + (cap * 16 + 255) // 256 * 256 + cap * 2 * 128 * 128 * 4


def test_compact_entry_points_reject_bad_arguments():
    L = cw.lib()
    p = cw.Pattern(20, 100, 2000, 2).c()
    assert L.cowa_compact_rows(None, 2) == 0
    # a band of ~2^31 positions has no compacted layout that an int row count can address
    wide = cw.Pattern(20, 2**31 - 1, 2000, 2).c()
    assert L.cowa_compact_rows(ctypes.byref(wide), 2) == 0
    assert L.cowa_compact_build(ctypes.byref(wide), 2, 100, 2, 128, _t(), _t(), 0x30000, 0x40000, None) == 2
    assert L.cowa_compact_append(ctypes.byref(wide), 2, 2, 128, 0x10000, 0x20000, 0x50000, 0x30000, 0x40000,
                                 None) == 2
    assert L.cowa_compact_append(ctypes.byref(p), 2, 2, 128, 0x10000, 0x20000, None, 0x30000, 0x40000, None) == 1
    assert L.cowa_compact_append(ctypes.byref(p), 2, 2, 96, 0x10000, 0x20000, 0x50000, 0x30000, 0x40000, None) == 2
    assert L.cowa_compact_build(ctypes.byref(p), 2, 100, 2, 128, _t(), _t(), 0x30008, 0x40000, None) == 3
    n = L.cowa_decode_compact_workspace_size(ctypes.byref(p), 2, 8, 2, 128)
    assert n > 256
    assert L.cowa_decode_compact(ctypes.byref(p), 2, 8, 2, 128, 0x10000, 0x30000, 0x40000, 0x50000, 0x60000, None,
                                 0x70000, n - 1, None) == 4


def test_fwd_varlen_rejects_bad_arguments_before_launch():
    L = cw.lib()
    p = cw.Pattern(64, 8, 1024, 4).c()
    n = L.cowa_fwd_varlen_workspace_size(ctypes.byref(p), 3, 1000, 8, 4, 128)
    assert n >= 256 + 16
    args = (ctypes.byref(p), 3, 1000, 8, 4, 128)
    assert L.cowa_fwd_varlen(*args, None, _t(), _t(), _t(), _t(), 0x20000, 0x40000, n, None) == 1      # no cu_seqlens
    assert L.cowa_fwd_varlen(*args, 0x30002, _t(), _t(), _t(), _t(), 0x20000, 0x40000, n, None) == 3   # misaligned
    assert L.cowa_fwd_varlen(*args, 0x30000, _t(), _t(), _t(), _t(), 0x20000, 0x40000, n - 1, None) == 4  # workspace
    assert L.cowa_fwd_varlen(ctypes.byref(p), 0, 1000, 8, 4, 128, 0x30000, _t(), _t(), _t(), _t(), 0x20000, 0x40000,
                             n, None) == 1                                                          # no sequences


def test_bwd_varlen_rejects_bad_arguments_before_launch():
    """The packed backward takes device cu_seqlens like the packed forward: the host checks what
    it can see (counts, pointers, alignment, workspace size) before anything is enqueued; the
    workspace holds the sequence table and the statistics of total/128 + n_seq tiles."""
    L = cw.lib()
    p = cw.Pattern(64, 8, 1024, 4).c()
    n = L.cowa_bwd_varlen_workspace_size(ctypes.byref(p), 3, 1000, 8, 4, 128)
    tiles = 1000 // 128 + 3
    assert n >= 256 + 4 * (3 * 3 + 1) + 2 * 8 * tiles * 128 * 4
    assert L.cowa_bwd_varlen_workspace_size(ctypes.byref(p), 6, 1000, 8, 4, 128) > n
    assert L.cowa_bwd_varlen_workspace_size(ctypes.byref(p), 3, 1000, 8, 4, 96) == 0
    assert L.cowa_bwd_varlen_workspace_size(ctypes.byref(p), 0, 1000, 8, 4, 128) == 0
    args = (ctypes.byref(p), 3, 1000, 8, 4, 128)

    def call(cu=0x30000, lse=0x20000, ws_bytes=n, n_seq=3):
        return L.cowa_bwd_varlen(ctypes.byref(p), n_seq, 1000, 8, 4, 128, cu, _t(), _t(), _t(), _t(), lse, _t(),
                                 _t(), _t(), _t(), 0x40000, ws_bytes, None)
    assert call(cu=None) == 1                 # no cu_seqlens
    assert call(cu=0x30002) == 3              # misaligned cu_seqlens
    assert call(lse=None) == 1                # no lse
    assert call(lse=0x20002) == 3             # misaligned lse
    assert call(ws_bytes=n - 1) == 4          # small workspace
    assert call(n_seq=0) == 1                 # no sequences
    bad = cw.c_tensor(0x10004, 1 << 20, 1024, 128)
    assert L.cowa_bwd_varlen(*args, 0x30000, _t(), _t(), _t(), _t(), 0x20000, bad, _t(), _t(), _t(), 0x40000, n,
                             None) == 3       # misaligned dO


def test_decode_and_bwd_reject_bad_arguments():
    L = cw.lib()
    p = cw.Pattern(64, 8, 1024, 4).c()
    # decode: null pos
    assert L.cowa_decode(ctypes.byref(p), 2, 8, 4, 128, 1024, 0x10000, _t(), _t(), None, 0x30000, None,
                         0x40000, 1 << 20, None) == 1
    # decode: small workspace
    assert L.cowa_decode(ctypes.byref(p), 2, 8, 4, 128, 1024, 0x10000, _t(), _t(), 0x50000, 0x30000, None,
                         0x40000, 8, None) == 4
    # bwd: misaligned dO
    assert L.cowa_bwd(ctypes.byref(p), 1, 128, 8, 4, 128, _t(), _t(), _t(), _t(), 0x20000,
                      cw.c_tensor(0x10004, 1 << 20, 1024, 128), _t(), _t(), _t(), 0x40000, 1 << 30, None) == 3
    assert L.cowa_fwd_workspace_size(ctypes.byref(p), 1, 128, 8, 4, 96) == 0
    assert L.cowa_decode_workspace_size(ctypes.byref(p), 16, 40, 8, 128, 131072) > 0


def test_status_strings():
    L = cw.lib()
    for s in range(7):
        assert len(L.cowa_status_string(s)) > 0
