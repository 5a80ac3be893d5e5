"""Pins for the CPU oracle: facts fixed by the pages and by mathematics.

Nothing here compares the oracle with itself.  Each test checks it against a
statement of the CoWA pages (union over heads = causal prefix, disjoint
intervals one per KV head, duplicated-window ablation at fixed widths), a
special case that reduces to a library routine (dense causal attention, SWA
with sinks), a brute-force scalar loop, a closed form, or finite differences.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import cowa_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# --------------------------------------------------------------------------
# mask and intervals
# --------------------------------------------------------------------------

PATTERN_GRID = [
    # (N, S, L, T, H)
    (64, 4, 8, 64, 4),
    (97, 0, 1, 97, 4),        # no sink, width-1 band, T-S not divisible by H
    (130, 7, 13, 130, 8),
    (200, 16, 5, 200, 3),
    (64, 64, 4, 64, 4),       # S = T: no long-range region
    (50, 3, 60, 50, 2),       # L > N
]


@pytest.mark.parametrize("N,S,L,T,H", PATTERN_GRID)
def test_union_over_heads_is_causal_prefix(N, S, L, T, H):
    """Every earlier token is visible to at least one KV head (N <= T, D = H)."""
    pat = orc.Pattern(S=S, L=L, T=T, D=H)
    rows = np.arange(N)
    union = np.zeros((N, N), bool)
    for g in range(H):
        union |= orc.visible_mask(rows, N, pat, g, H)
    assert np.array_equal(union, np.tril(np.ones((N, N), bool)))


@pytest.mark.parametrize("S,T,H", [(4, 64, 4), (0, 97, 4), (7, 130, 8), (16, 200, 3), (128, 32768, 8), (128, 131072, 8)])
def test_intervals_disjoint_cover_equal_width(S, T, H):
    """Non-overlapping long-range intervals, one per KV head, tiling [S, T) with equal widths."""
    pat = orc.Pattern(S=S, L=1, T=T, D=H)
    ivs = [orc.interval_of(G, pat, H) for G in range(H)]
    covered = np.zeros(T, int)
    for lo, hi in ivs:
        assert S <= lo <= hi <= T
        covered[lo:hi] += 1
    assert (covered[S:] == 1).all() and (covered[:S] == 0).all()
    widths = [hi - lo for lo, hi in ivs]
    assert max(widths) - min(widths) <= 1
    assert sum(widths) == T - S


def test_ablation_distinct_windows_fixed_width():
    """D distinct windows over 8 heads, widths fixed; only D = 8 covers everything."""
    gold = json.load(open(os.path.join(GOLDEN, "cowa_ablation_heads.json")))
    H = gold["h_kv"]
    S, T, N, L = 16, 16 + 8 * 40, 16 + 8 * 40, 8
    width_d8 = None
    for D, ndist in zip([1, 2, 4, 8], gold["distinct_windows"]):
        pat = orc.Pattern(S=S, L=L, T=T, D=D)
        ivs = [orc.interval_of(G, pat, H) for G in range(H)]
        assert len(set(ivs)) == ndist
        widths = {hi - lo for lo, hi in ivs}
        assert len(widths) == 1
        if width_d8 is None:
            width_d8 = widths.pop()
        else:
            assert widths.pop() == width_d8
        # heads whose global index agrees mod D see identical masks
        rows = np.arange(N)
        masks = [orc.visible_mask(rows, N, pat, g, H) for g in range(H)]
        for g in range(H):
            assert np.array_equal(masks[g], masks[g % D])
        union = np.zeros((N, N), bool)
        for m in masks:
            union |= m
        full = np.array_equal(union, np.tril(np.ones((N, N), bool)))
        assert full == (D == gold["full_collective_coverage_at"])
        # long-range coverage of [S, T) is the fraction D / H
        cov = np.zeros(T, bool)
        for lo, hi in ivs:
            cov[lo:hi] = True
        assert cov[S:].sum() == D * width_d8


def test_global_head_index_keeps_complementary_windows():
    """KV-head tensor parallelism: ranks holding heads [r*H/P, (r+1)*H/P) with the global
    index reproduce the single-device masks, so the union is still the causal prefix."""
    N, H, P = 96, 8, 4
    pat_full = orc.Pattern(S=4, L=6, T=N, D=H)
    rows = np.arange(N)
    ref = [orc.visible_mask(rows, N, pat_full, g, H) for g in range(H)]
    union = np.zeros((N, N), bool)
    for r in range(P):
        pat_r = orc.Pattern(S=4, L=6, T=N, D=H, kv_head_base=r * H // P, h_kv_global=H)
        for gl in range(H // P):
            m = orc.visible_mask(rows, N, pat_r, gl, H // P)
            assert np.array_equal(m, ref[r * H // P + gl])
            union |= m
    assert np.array_equal(union, np.tril(np.ones((N, N), bool)))


def _parse_ranges(txt):
    out = []
    for part in txt.split(","):
        a, b = part.split("-")
        out.extend(range(int(a), int(b) + 1))
    return out


def test_swa_with_sinks_golden():
    """T = S reduces CoWA to SWA(w, 4): 4 sink slots and w-4 recent slots (golden, by hand)."""
    pat = orc.Pattern(S=4, L=60, T=4, D=1)
    with open(os.path.join(GOLDEN, "swa_64_4.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            t, rng = line.split(":")
            t = int(t)
            want = _parse_ranges(rng.strip())
            got = np.nonzero(orc.visible_mask(np.array([t]), t + 1, pat, 0, 1)[0])[0].tolist()
            assert got == want, t


def test_small_cowa_layer_golden():
    """Visible sets of a 4-head layer (S=2, L=3, T=18; D=4 and the duplicated D=2) worked out by
    hand from the definition (golden), against the oracle's mask and the library's host counts."""
    from structured_sparse_attention_cowa_b200 import cowa as cw

    with open(os.path.join(GOLDEN, "cowa_small_visible.txt")) as f:
        rows = [ln for ln in f if ln.strip() and not ln.startswith("#")]
    assert len(rows) == 28
    for line in rows:
        head, rng = line.split(":")
        D, t, G = (int(x) for x in head.split())
        want = _parse_ranges(rng.strip())
        pat = orc.Pattern(S=2, L=3, T=18, D=D)
        got = np.nonzero(orc.visible_mask(np.array([t]), t + 1, pat, G, 4)[0])[0].tolist()
        assert got == want, (D, t, G)
        counts = cw.visible_counts(cw.Pattern(2, 3, 18, D), 4, 20)
        assert counts[G, t] == len(want), (D, t, G)


def _count_closed_form(t, S, L, lo, hi):
    """|sink U band U interval| at position t by inclusion-exclusion over three ranges."""
    def inter(*rs):
        a = max(r[0] for r in rs); b = min(r[1] for r in rs)
        return max(0, b - a)
    A = (0, min(S, t + 1))
    Bd = (max(0, t - L + 1), t + 1)
    C = (lo, min(hi, t + 1))
    return (inter(A) + inter(Bd) + inter(C) - inter(A, Bd) - inter(A, C) - inter(Bd, C)
            + inter(A, Bd, C))


def _vis_scalar(t, s, S, L, lo, hi):
    # written from the prose: causal, and in the sink, the L most recent keys, or the head's interval
    if s > t:
        return False
    return s < S or (t - s) < L or (lo <= s < hi)


@pytest.mark.parametrize("N,S,L,T,H,D", [(120, 5, 9, 120, 4, 4), (150, 0, 1, 140, 4, 2), (90, 12, 30, 90, 6, 3),
                                          (80, 10, 4, 40, 4, 4)])
def test_visible_counts_brute_force_and_closed_form(N, S, L, T, H, D):
    pat = orc.Pattern(S=S, L=L, T=T, D=D)
    counts = orc.visible_counts(N, pat, H)
    b = [S + (i * (T - S)) // H for i in range(H + 1)]
    for g in range(H):
        p = (g % D) * (H // D)
        lo, hi = b[p], b[p + 1]
        for t in range(N):
            brute = sum(_vis_scalar(t, s, S, L, lo, hi) for s in range(N))
            assert counts[g, t] == brute
            assert counts[g, t] == _count_closed_form(t, S, L, lo, hi)


# --------------------------------------------------------------------------
# forward values
# --------------------------------------------------------------------------

def test_dense_causal_special_case_matches_library_attention():
    """L >= T: every head sees the whole causal prefix -> textbook causal attention."""
    B, N, Hq, Hkv, d = 2, 40, 4, 2, 16
    q = rnd((B, N, Hq, d), 1); k = rnd((B, N, Hkv, d), 2); v = rnd((B, N, Hkv, d), 3)
    pat = orc.Pattern(S=3, L=N, T=N, D=Hkv)
    o, lse = orc.attention_fwd(q, k, v, pat)
    grp = Hq // Hkv
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(np.repeat(k, grp, axis=2)).permute(0, 2, 1, 3)
    vt = torch.from_numpy(np.repeat(v, grp, axis=2)).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)
    from scipy.special import logsumexp
    sc = np.einsum("bthd,bshd->bhts", q, np.repeat(k, grp, axis=2)) / math.sqrt(d)
    sc = np.where(np.tril(np.ones((N, N), bool)), sc, -np.inf)
    np.testing.assert_allclose(lse, logsumexp(sc, axis=-1), rtol=0, atol=1e-12)


def test_swa_special_case_matches_library_attention():
    """T = S: sink + sliding window (SWA with sinks) through a library attention with an explicit mask."""
    B, N, Hq, Hkv, d = 1, 70, 2, 1, 8
    w, nsink = 16, 4
    q = rnd((B, N, Hq, d), 4); k = rnd((B, N, Hkv, d), 5); v = rnd((B, N, Hkv, d), 6)
    pat = orc.Pattern(S=nsink, L=w - nsink, T=nsink, D=1)
    o, _ = orc.attention_fwd(q, k, v, pat)
    t = np.arange(N)[:, None]; s = np.arange(N)[None, :]
    swa = np.tril(np.ones((N, N), bool)) & ((s < nsink) | (np.triu(np.ones((N, N), bool), -(w - nsink - 1))))
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(np.repeat(k, Hq, axis=2)).permute(0, 2, 1, 3)
    vt = torch.from_numpy(np.repeat(v, Hq, axis=2)).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.from_numpy(swa))
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)


def test_first_row_and_constant_values():
    """Row t=0 sees only key 0: o = v_0, lse = scale q_0.k_0.  Constant V rows give o = v."""
    B, N, Hq, Hkv, d = 1, 33, 4, 2, 8
    pat = orc.Pattern(S=2, L=5, T=N, D=2)
    q = rnd((B, N, Hq, d), 7); k = rnd((B, N, Hkv, d), 8); v = rnd((B, N, Hkv, d), 9)
    o, lse = orc.attention_fwd(q, k, v, pat)
    for h in range(Hq):
        g = h // 2
        np.testing.assert_allclose(o[0, 0, h], v[0, 0, g], atol=1e-14)
        assert abs(lse[0, h, 0] - q[0, 0, h] @ k[0, 0, g] / math.sqrt(d)) < 1e-12
    vc = np.broadcast_to(rnd((1, 1, Hkv, d), 10), v.shape).copy()
    o2, _ = orc.attention_fwd(q, k, vc, pat)
    for h in range(Hq):
        np.testing.assert_allclose(o2[0, :, h], np.broadcast_to(vc[0, 0, h // 2], (N, d)), atol=1e-12)


def _brute_fwd(q, k, v, S, L, T, D):
    """Per-(b,h,t) scalar loops with math.exp, independent of the vectorised code."""
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]; grp = Hq // Hkv
    bnd = [S + (i * (T - S)) // Hkv for i in range(Hkv + 1)]
    sc = 1.0 / math.sqrt(d)
    o = np.zeros(q.shape); lse = np.zeros((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            g = h // grp
            p = (g % D) * (Hkv // D)
            lo, hi = bnd[p], bnd[p + 1]
            for t in range(N):
                keys = [s for s in range(N) if _vis_scalar(t, s, S, L, lo, hi)]
                scores = [sc * sum(q[b, t, h, x] * k[b, s, g, x] for x in range(d)) for s in keys]
                mx = max(scores)
                w = [math.exp(z - mx) for z in scores]
                den = sum(w)
                lse[b, h, t] = mx + math.log(den)
                for x in range(d):
                    o[b, t, h, x] = sum(wi * v[b, s, g, x] for wi, s in zip(w, keys)) / den
    return o, lse


@pytest.mark.parametrize("S,L,T,D", [(3, 4, 24, 2), (0, 1, 24, 1), (5, 30, 24, 2), (2, 3, 12, 2)])
def test_fwd_matches_brute_force_loops(S, L, T, D):
    B, N, Hq, Hkv, d = 1, 24, 4, 2, 4
    q = rnd((B, N, Hq, d), 11); k = rnd((B, N, Hkv, d), 12); v = rnd((B, N, Hkv, d), 13)
    pat = orc.Pattern(S=S, L=L, T=T, D=D)
    o, lse = orc.attention_fwd(q, k, v, pat)
    ob, lb = _brute_fwd(q, k, v, S, L, T, D)
    np.testing.assert_allclose(o, ob, atol=1e-12)
    np.testing.assert_allclose(lse, lb, atol=1e-12)


# --------------------------------------------------------------------------
# backward values
# --------------------------------------------------------------------------

@pytest.mark.parametrize("S,L,T,D", [(2, 3, 16, 2), (0, 16, 16, 1), (4, 1, 16, 2)])
def test_bwd_central_finite_differences(S, L, T, D):
    """Analytic gradients of sum(W*O) against central differences in fp64."""
    B, N, Hq, Hkv, d = 1, 16, 4, 2, 4
    q = rnd((B, N, Hq, d), 21); k = rnd((B, N, Hkv, d), 22); v = rnd((B, N, Hkv, d), 23)
    W = rnd((B, N, Hq, d), 24)
    pat = orc.Pattern(S=S, L=L, T=T, D=D)
    dq, dk, dv = orc.attention_bwd(q, k, v, W, pat)
    eps = 1e-6

    def f(args):
        return float((orc.attention_fwd(args["q"], args["k"], args["v"], pat)[0] * W).sum())

    for name, gx in (("q", dq), ("k", dk), ("v", dv)):
        base = {"q": q, "k": k, "v": v}
        x = base[name]
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp = x.copy(); xp[idx] += eps
            xm = x.copy(); xm[idx] -= eps
            num[idx] = (f({**base, name: xp}) - f({**base, name: xm})) / (2 * eps)
        rel = np.linalg.norm(num - gx) / np.linalg.norm(gx)
        assert rel < 1e-6, (name, rel)


def test_bwd_row_and_column_sum_identities():
    """Softmax rows sum to 1 and shifting all keys by a constant leaves the output unchanged:
    sum_s dv_g[s] = sum_{h in g} sum_t dO_h[t] and sum_s dk_g[s] = 0."""
    B, N, Hq, Hkv, d = 2, 48, 6, 2, 8
    q = rnd((B, N, Hq, d), 31); k = rnd((B, N, Hkv, d), 32); v = rnd((B, N, Hkv, d), 33)
    do = rnd((B, N, Hq, d), 34)
    pat = orc.Pattern(S=4, L=7, T=N, D=2)
    dq, dk, dv = orc.attention_bwd(q, k, v, do, pat)
    grp = Hq // Hkv
    for b in range(B):
        for g in range(Hkv):
            np.testing.assert_allclose(dv[b, :, g].sum(0), do[b, :, g * grp:(g + 1) * grp].sum((0, 1)), atol=1e-10)
            np.testing.assert_allclose(dk[b, :, g].sum(0), 0.0, atol=1e-10)


# --------------------------------------------------------------------------
# restricted evaluations, decode and tile plans
# --------------------------------------------------------------------------

def test_row_and_column_restricted_evaluation():
    B, N, Hq, Hkv, d = 1, 80, 4, 2, 8
    q = rnd((B, N, Hq, d), 41); k = rnd((B, N, Hkv, d), 42); v = rnd((B, N, Hkv, d), 43)
    do = rnd((B, N, Hq, d), 44)
    pat = orc.Pattern(S=5, L=9, T=N, D=2)
    o, lse = orc.attention_fwd(q, k, v, pat)
    rows = [0, 4, 5, 13, 40, 79]
    orow, lrow = orc.attention_fwd_rows(q, k, v, pat, rows, b=0)
    np.testing.assert_allclose(orow, o[0, rows], atol=1e-12)
    np.testing.assert_allclose(lrow, lse[0][:, rows].T, atol=1e-12)
    dq, dk, dv = orc.attention_bwd(q, k, v, do, pat)
    dqr = orc.attention_bwd_rows(q, k, v, do, pat, rows, b=0)
    np.testing.assert_allclose(dqr, dq[0, rows], atol=1e-10)
    cols = [0, 4, 6, 30, 44, 79]
    for g in range(Hkv):
        dkc, dvc = orc.attention_bwd_cols(q, k, v, do, pat, b=0, g=g, cols=cols, row_block=17)
        np.testing.assert_allclose(dkc, dk[0, cols, g], atol=1e-10)
        np.testing.assert_allclose(dvc, dv[0, cols, g], atol=1e-10)


def test_decode_is_row_pos_of_prefill():
    B, Hq, Hkv, d, Tc = 3, 4, 2, 8, 60
    kc = rnd((B, Hkv, Tc, d), 51); vc = rnd((B, Hkv, Tc, d), 52); qt = rnd((B, Hq, d), 53)
    pos = [59, 17, 0]
    pat = orc.Pattern(S=3, L=6, T=Tc, D=2)
    o, lse = orc.decode(qt, kc, vc, pos, pat)
    for b in range(B):
        t = pos[b]
        q = np.zeros((1, t + 1, Hq, d)); q[0, t] = qt[b]
        k = kc[b][:, : t + 1].transpose(1, 0, 2)[None]
        v = vc[b][:, : t + 1].transpose(1, 0, 2)[None]
        op, lp = orc.attention_fwd(q, k, v, pat)
        np.testing.assert_allclose(o[b], op[0, t], atol=1e-12)
        np.testing.assert_allclose(lse[b], lp[0, :, t], atol=1e-12)


@pytest.mark.parametrize("N,BM,BN,S,L,T,H,D", [(300, 32, 32, 16, 40, 300, 4, 4), (257, 64, 32, 0, 1, 250, 4, 2),
                                                (200, 16, 16, 20, 17, 120, 2, 2)])
def test_tile_plans_from_mask(N, BM, BN, S, L, T, H, D):
    """Every visible element is inside a visited tile, visited tiles hold one, full tiles hold only
    visible elements, and the backward plan is the transpose of the forward plan."""
    pat = orc.Pattern(S=S, L=L, T=T, D=D)
    fwd = orc.tile_plan_fwd(N, BM, BN, pat, H)
    bwd = orc.tile_plan_bwd(N, BM, BN, pat, H)
    b = [S + (i * (T - S)) // H for i in range(H + 1)]
    nq = -(-N // BM); nk = -(-N // BN)
    for g in range(H):
        p = (g % D) * (H // D); lo, hi = b[p], b[p + 1]
        for i in range(nq):
            visited = dict(fwd[(i, g)])
            for j in range(nk):
                els = [_vis_scalar(t, s, S, L, lo, hi) for t in range(i * BM, min(N, (i + 1) * BM))
                       for s in range(j * BN, min(N, (j + 1) * BN))]
                assert (j in visited) == any(els)
                if j in visited:
                    assert visited[j] == all(els)
                assert (i in bwd[(j, g)]) == (j in visited)


def test_bf16_widening_every_bit_pattern():
    """bf16_bits_to_f64 (how every GPU parity test hands the oracle the kernel's input bits)
    against torch's own bf16 -> float64 conversion for all 65,536 patterns, NaNs by class, and
    against values fixed by the bfloat16 format itself (1 sign, 8 exponent bits with bias 127,
    7 fraction bits: the upper half of an IEEE binary32)."""
    import torch

    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = orc.bf16_bits_to_f64(bits)
    want = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(want[~nan]))  # -0.0 keeps its sign
    landmarks = {0x3F80: 1.0, 0xC000: -2.0, 0x4049: 3.140625, 0x0001: 2.0 ** -133, 0x0080: 2.0 ** -126,
                 0x7F7F: (2 - 2.0 ** -7) * 2.0 ** 127, 0x7F80: np.inf, 0xFF80: -np.inf, 0x3E80: 0.25}
    for b, v in landmarks.items():
        assert orc.bf16_bits_to_f64(np.array([b], dtype=np.uint16))[0] == v, hex(b)
    assert np.signbit(orc.bf16_bits_to_f64(np.array([0x8000], dtype=np.uint16))[0])
