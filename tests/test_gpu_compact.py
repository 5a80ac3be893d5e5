"""GPU parity: decode over the compacted per-head cache (cowa_compact_build, cowa_compact_append,
cowa_decode_compact) against the fp64 oracle's decode over the full cache, and against
cowa_decode on the full cache.

Tolerances as for decode: o max-abs <= 2e-2, lse max-abs <= 1e-3 against fp64 on identical bf16
inputs."""

import numpy as np
import pytest
import torch

from oracle import cowa_oracle as orc
from structured_sparse_attention_cowa_b200 import cowa as cw
from structured_sparse_attention_cowa_b200 import synth
from tests.gpu_helpers import LSE_ATOL, O_ATOL, host_and_device, oracle_pattern, to64

pytestmark = pytest.mark.gpu


def _full_cache_views(k64, v64):
    """[B, N, H_kv, d] float64 arrays -> the oracle's [B, H_kv, T, d] cache layout."""
    return np.ascontiguousarray(k64.transpose(0, 2, 1, 3)), np.ascontiguousarray(v64.transpose(0, 2, 1, 3))


def _check(o, lse, want_o, want_l, what):
    err_o = np.abs(to64(o) - want_o).max()
    err_l = np.abs(lse.cpu().numpy().astype(np.float64) - want_l).max()
    assert err_o <= O_ATOL and err_l <= LSE_ATOL, (what, err_o, err_l)


@pytest.mark.parametrize("Hq,Hkv,d,pat", [
    (8, 2, 128, cw.Pattern(20, 100, 2000, 2)),      # S, L not multiples of 64
    (10, 2, 128, cw.Pattern(64, 256, 1500, 1)),     # duplicated windows (D = 1), group of 5
    (8, 4, 64, cw.Pattern(0, 70, 1800, 4)),         # no sink, d = 64
    (4, 2, 128, cw.Pattern(16, 90, 16, 2)),         # SWA + sinks (T = S): no interval region
])
def test_decode_compact_after_build(cuda_device, Hq, Hkv, d, pat):
    """Compacted cache built from a 1500-token prefill, decode of a new query at several
    positions of the prefill (every position's own K/V present)."""
    B, N = 2, 1500
    k64, k = host_and_device((B, N, Hkv, d), "k", cuda_device, 21)
    v64, v = host_and_device((B, N, Hkv, d), "v", cuda_device, 21)
    qt64, qt = host_and_device((B, Hq, d), "q_t", cuda_device, 21)
    kf, vf = _full_cache_views(k64, v64)
    for last in (N - 1, 1300):
        # rebuild for a shorter history so the band ring ends at `last`
        kc, vc = cw.compact_cache(k[:, :last + 1], v[:, :last + 1], pat)
        pos = torch.tensor([last, last], dtype=torch.int32, device=cuda_device)
        o, lse = cw.cowa_decode_compact(qt, kc, vc, pos, pat)
        torch.cuda.synchronize()
        want_o, want_l = orc.decode(qt64, kf, vf, [last, last], oracle_pattern(pat))
        _check(o, lse, want_o, want_l, ("build", last))
        # and the full-cache decode on the same data
        o2, lse2 = cw.cowa_decode(qt, k.transpose(1, 2), v.transpose(1, 2), pos, pat)
        assert np.abs(to64(o) - to64(o2)).max() <= O_ATOL
        assert float((lse - lse2).abs().max()) <= LSE_ATOL


def test_decode_compact_append_sequence(cuda_device):
    """Prefill of 12 tokens, then one append + decode per token up to position 1150: appends
    cross the sink end (S = 20), the band ring wraps every R rows, head 1's interval starts at
    1010; B = 2 sequences at different positions (the second lags by 7 tokens)."""
    B, Hq, Hkv, d = 2, 8, 2, 128
    pat = cw.Pattern(20, 100, 2000, 2)
    N, N0, lag = 1151, 12, 7
    k64, k = host_and_device((B, N, Hkv, d), "k", cuda_device, 23)
    v64, v = host_and_device((B, N, Hkv, d), "v", cuda_device, 23)
    qt64, qt = host_and_device((B, Hq, d), "q_t", cuda_device, 23)
    kf, vf = _full_cache_views(k64, v64)
    kc, vc = cw.compact_cache(k[:, :N0], v[:, :N0], pat)
    check_at = set(range(N0, 40)) | set(range(N0, N, 37)) | {1009, 1010, 1011, N - 1}
    ws = torch.zeros(cw.lib().cowa_decode_compact_workspace_size(
        __import__("ctypes").byref(pat.c()), B, Hq, Hkv, d), dtype=torch.uint8, device=cuda_device)
    for p in range(N0, N + lag):
        pos_l = [p if p < N else -1, p - lag if p - lag >= N0 else -1]  # -1: no append for that row
        pos = torch.tensor(pos_l, dtype=torch.int32, device=cuda_device)
        idx = torch.tensor([max(x, 0) for x in pos_l], device=cuda_device)
        k_new = k[torch.arange(B, device=cuda_device), idx]   # [B, H_kv, d]
        v_new = v[torch.arange(B, device=cuda_device), idx]
        cw.compact_append(kc, vc, k_new, v_new, pos, pat)
        if p in check_at and p < N:
            pos_d = torch.tensor([p, max(p - lag, N0 - 1)], dtype=torch.int32, device=cuda_device)
            o, lse = cw.cowa_decode_compact(qt, kc, vc, pos_d, pat, workspace=ws)
            torch.cuda.synchronize()
            want_o, want_l = orc.decode(qt64, kf, vf, pos_d.tolist(), oracle_pattern(pat))
            _check(o, lse, want_o, want_l, ("append", p))
    assert cw.workspace_status(ws) == 0


def test_decode_compact_128k_config_matches_full_cache(cuda_device):
    """The 128K decode configuration (S=128, L=4096, T=131072, D=8) at 4 sequences: the compacted
    cache (20,736 rows per head instead of 131,072) gives the full-cache decode's result."""
    B, Hq, Hkv, d, T = 4, 40, 8, 128, 131072
    pat = cw.Pattern(128, 4096, 131072, 8)
    assert cw.compact_rows(pat, Hkv) == 20736
    k = synth.cuda_normal_bf16((B, T, Hkv, d), synth.seed_of("k_cache"), cuda_device)
    v = synth.cuda_normal_bf16((B, T, Hkv, d), synth.seed_of("v_cache"), cuda_device)
    qt = synth.cuda_normal_bf16((B, Hq, d), synth.seed_of("q_t"), cuda_device)
    kc, vc = cw.compact_cache(k, v, pat)
    pos = torch.full((B,), T - 1, dtype=torch.int32, device=cuda_device)
    o, lse = cw.cowa_decode_compact(qt, kc, vc, pos, pat)
    o2, lse2 = cw.cowa_decode(qt, k.transpose(1, 2), v.transpose(1, 2), pos, pat)
    torch.cuda.synchronize()
    assert float((o.float() - o2.float()).abs().max()) <= O_ATOL
    assert float((lse - lse2).abs().max()) <= LSE_ATOL
