"""GPU parity: KV-head tensor parallelism with the ranks' calls made one after another on one GPU.

The layer's KV heads are split over P ranks (shard.kv_head_runs); every run of consecutive global
heads is one cowa_fwd / cowa_bwd / cowa_decode call on that run's heads only, with the run's
kv_head_base and the layer's h_kv_global.  Each run's results are compared with the fp64 oracle
over the whole (unsplit) layer, restricted to the run's heads.  The calls do not wait on one
another: the op has no exchange step between ranks."""

import numpy as np
import pytest
import torch

from oracle import cowa_oracle as orc
from structured_sparse_attention_cowa_b200 import cowa as cw
from structured_sparse_attention_cowa_b200 import shard
from structured_sparse_attention_cowa_b200 import synth
from tests.gpu_helpers import GRAD_RTOL, LSE_ATOL, O_ATOL, grad_bounds, grad_errors, host_and_device, oracle_pattern, to64

pytestmark = pytest.mark.gpu


def _heads(x, r: range):
    return x[:, :, r.start:r.stop].contiguous()


@pytest.mark.parametrize("P,order", [(2, "folded"), (4, "contiguous")])
def test_tp_prefill_runs_reproduce_the_layer(cuda_device, P, order):
    B, N, Hq, Hkv, d = 1, 700, 8, 4, 128
    grp = Hq // Hkv
    pat = cw.Pattern(24, 50, 640, 4)
    q64, q = host_and_device((B, N, Hq, d), "q", cuda_device, 31)
    k64, k = host_and_device((B, N, Hkv, d), "k", cuda_device, 31)
    v64, v = host_and_device((B, N, Hkv, d), "v", cuda_device, 31)
    do64, do = host_and_device((B, N, Hq, d), "do", cuda_device, 31)
    op = oracle_pattern(pat)
    wo, wl = orc.attention_fwd(q64, k64, v64, op)
    wq, wk, wv = orc.attention_bwd(q64, k64, v64, do64, op)
    covered = []
    for r in range(P):
        for run in shard.kv_head_runs(r, P, Hkv, grp, order):
            qh, kh = run.q_heads, run.kv_heads
            rp = shard.run_pattern(pat, run, Hkv)
            qr, kr, vr, dor = _heads(q, qh), _heads(k, kh), _heads(v, kh), _heads(do, qh)
            o, lse = cw.cowa_fwd(qr, kr, vr, rp)
            dq, dk, dv = cw.cowa_bwd(qr, kr, vr, o, lse, dor, rp)
            torch.cuda.synchronize()
            qs, ks = slice(qh.start, qh.stop), slice(kh.start, kh.stop)
            assert np.abs(to64(o) - wo[:, :, qs]).max() <= O_ATOL, (r, run)
            assert np.abs(lse.cpu().numpy() - wl[:, qs]).max() <= LSE_ATOL, (r, run)
            bounds = grad_bounds(q64[:, :, qs], k64[:, :, ks], v64[:, :, ks], do64[:, :, qs], op.sm_scale(d))
            errs = grad_errors((to64(dq), to64(dk), to64(dv)), (wq[:, :, qs], wk[:, :, ks], wv[:, :, ks]), bounds)
            assert max(errs) <= GRAD_RTOL, (r, run, errs)
            covered += list(kh)
    assert sorted(covered) == list(range(Hkv))


def test_tp_decode_runs_reproduce_the_layer(cuda_device):
    B, Hq, Hkv, d, T_cap = 4, 8, 4, 128, 1024
    grp = Hq // Hkv
    pat = cw.Pattern(64, 128, 1024, 4)
    pos = [1023, 700, 64, 0]
    kc64, kc = host_and_device((B, Hkv, T_cap, d), "k_cache", cuda_device, 31)
    vc64, vc = host_and_device((B, Hkv, T_cap, d), "v_cache", cuda_device, 31)
    qt64, qt = host_and_device((B, Hq, d), "q_t", cuda_device, 31)
    want_o, want_l = orc.decode(qt64, kc64, vc64, pos, oracle_pattern(pat))
    pos_t = torch.tensor(pos, dtype=torch.int32, device=cuda_device)
    for r in range(2):
        for run in shard.kv_head_runs(r, 2, Hkv, grp, "folded"):
            qh, kh = run.q_heads, run.kv_heads
            o, lse = cw.cowa_decode(qt[:, qh.start:qh.stop].contiguous(), kc[:, kh.start:kh.stop].contiguous(),
                                    vc[:, kh.start:kh.stop].contiguous(), pos_t, shard.run_pattern(pat, run, Hkv))
            torch.cuda.synchronize()
            assert np.abs(to64(o) - want_o[:, qh.start:qh.stop]).max() <= O_ATOL, (r, run)
            assert np.abs(lse.cpu().numpy() - want_l[:, qh.start:qh.stop]).max() <= LSE_ATOL, (r, run)


@pytest.mark.parametrize("g", [0, 7])
def test_tp_rank_of_one_kv_head_at_32k_matches_the_layer(cuda_device, g):
    """A rank holding one KV head of the 32K layer (H_q = 40, H_kv = 8, S = 128, L = 2048): its
    backward call splits the long key tiles (head 0: 121 chunks, head 7: 13) and reproduces
    that head of the unsplit 8-head call.  dq is the same kernel on the same rows (equal bits);
    dk, dv differ only by the fp32 order of the chunks' partial sums (bf16 rounding)."""
    import ctypes

    B, N, Hq, Hkv, d = 1, 32768, 40, 8, 128
    grp = Hq // Hkv
    q, k, v, do = (synth.cuda_normal_bf16(s, synth.seed_of(n, 41), cuda_device)
                   for s, n in (((B, N, Hq, d), "q"), ((B, N, Hkv, d), "k"), ((B, N, Hkv, d), "v"),
                                ((B, N, Hq, d), "do")))
    layer = cw.Pattern(128, 2048, 32768, 8)
    o, lse = cw.cowa_fwd(q, k, v, layer)
    dq, dk, dv = cw.cowa_bwd(q, k, v, o, lse, do, layer)
    one = cw.Pattern(128, 2048, 32768, 8, kv_head_base=g, h_kv_global=8)
    hq = slice(g * grp, (g + 1) * grp)
    qg, kg, vg, dog = (x.contiguous() for x in (q[:, :, hq], k[:, :, g:g + 1], v[:, :, g:g + 1], do[:, :, hq]))
    og, lseg = cw.cowa_fwd(qg, kg, vg, one)
    assert torch.equal(og, o[:, :, hq]) and torch.equal(lseg, lse[:, hq])
    L = cw.lib()
    n_ws = L.cowa_bwd_workspace_size(ctypes.byref(one.c()), B, N, grp, 1, d)
    assert n_ws > 256 + 2 * grp * N * 4  # the call splits its long key tiles
    ws = torch.zeros(n_ws, dtype=torch.uint8, device=cuda_device)
    dqg, dkg, dvg = cw.cowa_bwd(qg, kg, vg, og, lseg, dog, one, workspace=ws)
    torch.cuda.synchronize()
    assert cw.workspace_status(ws) == 0
    assert torch.equal(dqg, dq[:, :, hq])
    for got, want in ((dkg, dk[:, :, g:g + 1]), (dvg, dv[:, :, g:g + 1])):
        a, b = got.float(), want.float()
        rel = float((a - b).norm() / b.norm())
        assert rel <= 2e-3, rel
        assert float((a == b).float().mean()) >= 0.9  # most elements round to the same bf16
