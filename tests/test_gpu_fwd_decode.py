"""GPU parity: cowa_fwd and cowa_decode (through the C ABI) against the fp64 oracle.

Tolerances: o max-abs <= 2e-2, lse max-abs <= 1e-3 against fp64 on identical bf16 inputs;
tile plans bit-exact."""

import numpy as np
import pytest
import torch

from oracle import cowa_oracle as orc
from structured_sparse_attention_cowa_b200 import cowa as cw
from structured_sparse_attention_cowa_b200 import synth
from tests.gpu_helpers import (LSE_ATOL, O_ATOL, DeviceView, edge_rows, host_and_device, oracle_pattern, to64)

pytestmark = pytest.mark.gpu


def _check_fwd_full(B, N, Hq, Hkv, d, pat, device, extra=0):
    q64, q = host_and_device((B, N, Hq, d), "q", device, extra)
    k64, k = host_and_device((B, N, Hkv, d), "k", device, extra)
    v64, v = host_and_device((B, N, Hkv, d), "v", device, extra)
    o, lse = cw.cowa_fwd(q, k, v, pat)
    torch.cuda.synchronize()
    want_o, want_l = orc.attention_fwd(q64, k64, v64, oracle_pattern(pat))
    err_o = np.abs(to64(o) - want_o).max()
    err_l = np.abs(lse.cpu().numpy().astype(np.float64) - want_l).max()
    assert err_o <= O_ATOL and err_l <= LSE_ATOL, (err_o, err_l)


def test_device_plan_matches_host_plan(cuda_device):
    for N, Hkv, pat in [(1024, 4, cw.Pattern(64, 128, 1024, 4)), (8192, 8, cw.Pattern(128, 1024, 8192, 2)),
                        (1000, 3, cw.Pattern(0, 1, 900, 3))]:
        host = sorted(map(tuple, cw.plan_debug(pat, Hkv, N, 128, 128, 0).tolist()))
        dev = sorted(map(tuple, cw.plan_debug(pat, Hkv, N, 128, 128, 2).tolist()))
        assert host == dev


@pytest.mark.parametrize("D", [4, 2, 1])
def test_fwd_tiny_config(cuda_device, D):
    """B=1, N=T=1024, H_q=8, H_kv=4, d=64, S=64, L=128; D=4 plus the duplicated D=2, 1."""
    _check_fwd_full(1, 1024, 8, 4, 64, cw.Pattern(64, 128, 1024, D), cuda_device)


@pytest.mark.parametrize("B,N,Hq,Hkv,d,pat", [
    (1, 1000, 10, 2, 128, cw.Pattern(64, 128, 1000, 2)),     # ragged tail, odd group of 5
    (2, 333, 4, 4, 128, cw.Pattern(5, 40, 333, 4)),          # group of 1, tile-unaligned sink
    (1, 77, 6, 2, 64, cw.Pattern(0, 1, 77, 2)),              # single partial tile, L = 1
    (1, 640, 8, 2, 128, cw.Pattern(16, 640, 640, 2)),        # dense causal (L >= T)
    (1, 520, 4, 2, 64, cw.Pattern(4, 60, 4, 1)),             # SWA + sinks (T = S)
    (1, 700, 8, 4, 128, cw.Pattern(32, 100, 500, 4)),        # N > T
    (1, 300, 2, 1, 128, cw.Pattern(7, 30, 300, 2, kv_head_base=1, h_kv_global=2)),  # TP rank 1 of 2
    (1, 256, 16, 2, 64, cw.Pattern(16, 64, 256, 2, softmax_scale=0.3)),  # group of 8, explicit scale
    (1, 700, 8, 4, 128, cw.Pattern(16, 50, 2**31 - 1, 4)),   # declared span of INT_MAX: intervals past N
    (1, 300, 4, 2, 64, cw.Pattern(2**31 - 1, 1, 2**31 - 1, 2)),  # sink of INT_MAX: dense causal
])
def test_fwd_edge_shapes(cuda_device, B, N, Hq, Hkv, d, pat):
    _check_fwd_full(B, N, Hq, Hkv, d, pat, cuda_device, extra=1)


def test_fwd_strided_inputs(cuda_device):
    """q, k, v as views into one packed [B, N, Hq + 2 Hkv, d] buffer; o written into a strided view."""
    B, N, Hq, Hkv, d = 1, 500, 8, 2, 128
    pat = cw.Pattern(32, 64, 500, 2)
    qkv64, qkv = host_and_device((B, N, Hq + 2 * Hkv, d), "q", cuda_device, 7)
    q, k, v = qkv[:, :, :Hq], qkv[:, :, Hq:Hq + Hkv], qkv[:, :, Hq + Hkv:]
    obuf = torch.zeros((B, N, 2 * Hq, d), dtype=torch.bfloat16, device=cuda_device)
    o, lse = cw.cowa_fwd(q, k, v, pat, out=obuf[:, :, Hq:])
    want_o, want_l = orc.attention_fwd(qkv64[:, :, :Hq], qkv64[:, :, Hq:Hq + Hkv], qkv64[:, :, Hq + Hkv:],
                                       oracle_pattern(pat))
    assert np.abs(to64(obuf[:, :, Hq:]) - want_o).max() <= O_ATOL
    assert float(obuf[:, :, :Hq].abs().max()) == 0.0
    assert np.abs(lse.cpu().numpy() - want_l).max() <= LSE_ATOL


def test_fwd_running_max_growth(cuda_device):
    """Scores that jump in a later tile: keys of some tiles scaled up so that the running row
    max grows by far more than the lazy-rescale threshold after the first tile (rescale of O
    and a redone tile), next to the reverse case (large sink keys: no growth after tile 0)."""
    B, N, Hq, Hkv, d = 1, 1000, 4, 2, 128
    pat = cw.Pattern(16, 512, 1000, 2)
    q64, q = host_and_device((B, N, Hq, d), "q", cuda_device, 11)
    _, k = host_and_device((B, N, Hkv, d), "k", cuda_device, 11)
    v64, v = host_and_device((B, N, Hkv, d), "v", cuda_device, 11)
    for lo, hi, f in [(768, 1000, 6.0), (0, 16, 6.0), (300, 420, 4.0)]:
        k2 = k.clone()
        k2[:, lo:hi] = (k2[:, lo:hi].float() * f).to(torch.bfloat16)
        o, lse = cw.cowa_fwd(q, k2, v, pat)
        torch.cuda.synchronize()
        want_o, want_l = orc.attention_fwd(q64, to64(k2), v64, oracle_pattern(pat))
        err_o = np.abs(to64(o) - want_o).max()
        err_l = np.abs(lse.cpu().numpy().astype(np.float64) - want_l).max()
        assert err_o <= O_ATOL and err_l <= LSE_ATOL, (lo, hi, err_o, err_l)


@pytest.mark.parametrize("d", [128, 64])
def test_fwd_chunked_prefill(cuda_device, d):
    """Query blocks at offsets 0, 300, 700 of a 1000-token prefill (ragged, not tile-aligned)
    against the keys written so far: each block equals the oracle's rows and the one-pass
    forward's rows; keys past the block (present or not) change nothing."""
    B, N, Hq, Hkv = 1, 1000, 10, 2
    pat = cw.Pattern(64, 128, 1000, 2)
    q64, q = host_and_device((B, N, Hq, d), "q", cuda_device, 13)
    k64, k = host_and_device((B, N, Hkv, d), "k", cuda_device, 13)
    v64, v = host_and_device((B, N, Hkv, d), "v", cuda_device, 13)
    want_o, want_l = orc.attention_fwd(q64, k64, v64, oracle_pattern(pat))
    full_o, full_l = cw.cowa_fwd(q, k, v, pat)
    for lo, hi, n_k in [(0, 300, 300), (300, 700, 1000), (700, 1000, 1000), (640, 1000, 1000)]:
        o, lse = cw.cowa_fwd_chunk(q[:, lo:hi].contiguous(), k, v, pat, q_offset=lo, n_k=n_k)
        torch.cuda.synchronize()
        err_o = np.abs(to64(o) - want_o[:, lo:hi]).max()
        err_l = np.abs(lse.cpu().numpy().astype(np.float64) - want_l[:, :, lo:hi]).max()
        assert err_o <= O_ATOL and err_l <= LSE_ATOL, (lo, hi, err_o, err_l)
        assert np.abs(to64(o) - to64(full_o[:, lo:hi])).max() <= O_ATOL
        assert float((lse - full_l[:, :, lo:hi]).abs().max()) <= LSE_ATOL


def test_fwd_chunked_prefill_over_a_kv_cache(cuda_device):
    """The block's keys come from a [B, H_kv, T_cap, d] cache (as decode uses) holding the first
    n_k positions and unrelated data after them: B=2, a 360-row block at offset 640."""
    B, N, Hq, Hkv, d, T_cap = 2, 1000, 8, 4, 128, 1152
    pat = cw.Pattern(32, 200, 1000, 4)
    q64, q = host_and_device((B, N, Hq, d), "q", cuda_device, 17)
    k64, k = host_and_device((B, N, Hkv, d), "k", cuda_device, 17)
    v64, v = host_and_device((B, N, Hkv, d), "v", cuda_device, 17)
    kc = synth.cuda_normal_bf16((B, Hkv, T_cap, d), 99, cuda_device)
    vc = synth.cuda_normal_bf16((B, Hkv, T_cap, d), 98, cuda_device)
    kc[:, :, :N] = k.transpose(1, 2)
    vc[:, :, :N] = v.transpose(1, 2)
    lo, hi = 640, 1000
    o, lse = cw.cowa_fwd_chunk(q[:, lo:hi].contiguous(), kc, vc, pat, q_offset=lo, n_k=N, kv_layout="bhtd")
    torch.cuda.synchronize()
    want_o, want_l = orc.attention_fwd(q64, k64, v64, oracle_pattern(pat))
    assert np.abs(to64(o) - want_o[:, lo:hi]).max() <= O_ATOL
    assert np.abs(lse.cpu().numpy().astype(np.float64) - want_l[:, :, lo:hi]).max() <= LSE_ATOL


def test_fwd_chunked_prefill_8k(cuda_device):
    """Prefill 8K shapes (H_q=32, H_kv=8, S=128, L=1024, D=8): the block [4096, 6144) against
    keys 0..6143, every row of batch 0 against the oracle."""
    B, N, Hq, Hkv, d = 1, 8192, 32, 8, 128
    pat = cw.Pattern(128, 1024, 8192, 8)
    qh, q = host_and_device((B, N, Hq, d), "q", cuda_device)
    kh, k = host_and_device((B, N, Hkv, d), "k", cuda_device)
    vh, v = host_and_device((B, N, Hkv, d), "v", cuda_device)
    lo, hi = 4096, 6144
    o, lse = cw.cowa_fwd_chunk(q[:, lo:hi].contiguous(), k, v, pat, q_offset=lo, n_k=hi)
    torch.cuda.synchronize()
    rows = np.arange(lo, hi)
    want_o, want_l = orc.attention_fwd_rows(qh, kh, vh, oracle_pattern(pat), rows, b=0)
    assert np.abs(to64(o[0]) - want_o).max() <= O_ATOL
    assert np.abs(lse[0].T.cpu().numpy().astype(np.float64) - want_l).max() <= LSE_ATOL


def _check_fwd_rows(B, N, Hq, Hkv, d, pat, device, rows, batches, use_cuda_gen=False):
    if use_cuda_gen:
        q = synth.cuda_normal_bf16((B, N, Hq, d), synth.seed_of("q"), device)
        k = synth.cuda_normal_bf16((B, N, Hkv, d), synth.seed_of("k"), device)
        v = synth.cuda_normal_bf16((B, N, Hkv, d), synth.seed_of("v"), device)
        qh, kh, vh = DeviceView(q), DeviceView(k), DeviceView(v)
    else:
        qh, q = host_and_device((B, N, Hq, d), "q", device)
        kh, k = host_and_device((B, N, Hkv, d), "k", device)
        vh, v = host_and_device((B, N, Hkv, d), "v", device)
    o, lse = cw.cowa_fwd(q, k, v, pat)
    torch.cuda.synchronize()
    rows_t = torch.as_tensor(rows, device=device)
    for b in batches:
        want_o, want_l = orc.attention_fwd_rows(qh, kh, vh, oracle_pattern(pat), rows, b=b)
        got_o = to64(o[b, rows_t])
        got_l = lse[b][:, rows_t].T.cpu().numpy().astype(np.float64)
        err_o = np.abs(got_o - want_o).max()
        err_l = np.abs(got_l - want_l).max()
        assert err_o <= O_ATOL and err_l <= LSE_ATOL, (b, err_o, err_l)


def test_fwd_prefill_8k_full(cuda_device):
    """B=2, N=T=8192, H_q=32, H_kv=8, d=128, S=128, L=1024, D=8: every row of batch 0."""
    pat = cw.Pattern(128, 1024, 8192, 8)
    _check_fwd_rows(2, 8192, 32, 8, 128, pat, cuda_device, np.arange(8192), batches=[0])


@pytest.mark.parametrize("D", [4, 2, 1])
def test_fwd_prefill_8k_window_matched_sweep(cuda_device, D):
    pat = cw.Pattern(128, 1024, 8192, D)
    rows = edge_rows(8192, pat, 8, extra_random=256, seed=D)
    _check_fwd_rows(2, 8192, 32, 8, 128, pat, cuda_device, rows, batches=[0, 1])


def test_fwd_train_32k_sampled_rows(cuda_device):
    """B=1, N=T=32768, H_q=40, H_kv=8, d=128, S=128, L=2048, D=8 (sampled rows, all heads)."""
    pat = cw.Pattern(128, 2048, 32768, 8)
    rows = edge_rows(32768, pat, 8, extra_random=512, seed=3)
    _check_fwd_rows(1, 32768, 40, 8, 128, pat, cuda_device, rows, batches=[0], use_cuda_gen=True)


def test_fwd_long_128k_sampled_rows(cuda_device):
    """B=1, N=T=131072, H_q=40, H_kv=8, d=128, S=128, L=4096, D=8 and its dense-causal mode."""
    for pat in (cw.Pattern(128, 4096, 131072, 8), cw.Pattern(128, 131072, 131072, 8)):
        rows = edge_rows(131072, pat, 8, extra_random=64, seed=4)
        if pat.L >= 131072:
            rows = np.array(sorted(set(rows.tolist()) - set(range(2, 131000)) | {65536, 99999}))
        _check_fwd_rows(1, 131072, 40, 8, 128, pat, cuda_device, rows, batches=[0], use_cuda_gen=True)
        torch.cuda.empty_cache()


# ----------------------------------------------------------------------------------- decode
def _check_decode(B, Hq, Hkv, d, T_cap, pat, pos, device, layout="bhtd", sample_b=None, cuda_gen=False):
    shape = (B, Hkv, T_cap, d) if layout == "bhtd" else (B, T_cap, Hkv, d)
    if cuda_gen:
        kc = synth.cuda_normal_bf16(shape, synth.seed_of("k_cache"), device)
        vc = synth.cuda_normal_bf16(shape, synth.seed_of("v_cache"), device)
        qt64, qt = host_and_device((B, Hq, d), "q_t", device)
    else:
        _, kc = host_and_device(shape, "k_cache", device)
        _, vc = host_and_device(shape, "v_cache", device)
        qt64, qt = host_and_device((B, Hq, d), "q_t", device)
    pos_t = torch.tensor(pos, dtype=torch.int32, device=device)
    o, lse = cw.cowa_decode(qt, kc, vc, pos_t, pat, layout=layout)
    torch.cuda.synchronize()
    kv = DeviceView(kc if layout == "bhtd" else kc.permute(0, 2, 1, 3))
    vv = DeviceView(vc if layout == "bhtd" else vc.permute(0, 2, 1, 3))
    bs = range(B) if sample_b is None else sample_b
    for b in bs:
        want_o, want_l = orc.decode(qt64[b:b + 1], _Slice(kv, b), _Slice(vv, b), [pos[b]], oracle_pattern(pat))
        err_o = np.abs(to64(o[b]) - want_o[0]).max()
        err_l = np.abs(lse[b].cpu().numpy().astype(np.float64) - want_l[0]).max()
        assert err_o <= O_ATOL and err_l <= LSE_ATOL, (b, pos[b], err_o, err_l)


class _Slice:
    """Batch b of a DeviceView, presented as a batch of one."""

    def __init__(self, view, b):
        self.view, self.b = view, b
        self.shape = (1,) + view.shape[1:]

    def __getitem__(self, idx):
        return self.view[(self.b,) + tuple(idx[1:])]


@pytest.mark.parametrize("d,Hq,Hkv", [(64, 8, 4), (128, 8, 4), (128, 10, 2), (128, 8, 8), (64, 16, 2)])
def test_decode_small(cuda_device, d, Hq, Hkv):
    T_cap = 1024
    pat = cw.Pattern(64, 128, 1024, Hkv)
    pos = [0, 63, 64, 200, 1023, 511]
    _check_decode(len(pos), Hq, Hkv, d, T_cap, pat, pos, cuda_device)


@pytest.mark.parametrize("pat", [cw.Pattern(16, 50, 2**31 - 1, 4),         # intervals far past the cache
                                 cw.Pattern(8, 2**31 - 1, 1024, 4),          # window of INT_MAX (dense)
                                 cw.Pattern(2**31 - 1, 1, 2**31 - 1, 4)])    # every key a sink key
def test_decode_extreme_patterns(cuda_device, pat):
    """Pattern parameters at the int range's end: plans and chunking stay exact."""
    pos = [0, 127, 640, 1023]
    _check_decode(len(pos), 8, 4, 128, 1024, pat, pos, cuda_device)


def test_decode_token_major_cache_and_duplicated_windows(cuda_device):
    pat = cw.Pattern(16, 100, 2000, 2)
    pos = [1999, 17, 1500, 100]
    _check_decode(4, 8, 4, 128, 2048, pat, pos, cuda_device, layout="bthd")


def test_decode_128k_config(cuda_device):
    """B=16 sequences, cache 131072 tokens, H_q=40, H_kv=8, d=128, pos=131071, S=128, L=4096, D=8;
    sampled sequences against the oracle."""
    B = 16
    pat = cw.Pattern(128, 4096, 131072, 8)
    pos = [131071] * B
    pos[3] = 70000
    pos[5] = 4000
    _check_decode(B, 40, 8, 128, 131072, pat, pos, cuda_device, sample_b=[0, 3, 5, 15], cuda_gen=True)


def test_device_wait_timeout_is_reported_and_context_survives(cuda_device):
    """A device-side wait that runs out sets the workspace status word; the kernel returns, the
    host reads COWA_ERR_TIMEOUT, and the next call on the same context is correct."""
    import ctypes
    ws = torch.zeros(256, dtype=torch.uint8, device=cuda_device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert cw.lib().cowa_debug_wait_timeout(ctypes.c_void_p(ws.data_ptr()), 256, 50_000_000, stream) == 0
    assert cw.workspace_status(ws) == 6          # COWA_ERR_TIMEOUT, and the word is cleared
    assert cw.workspace_status(ws) == 0
    _check_fwd_full(1, 300, 4, 2, 64, cw.Pattern(8, 32, 300, 2), cuda_device, extra=5)


def test_fwd_varlen_packed_batch(cuda_device):
    """Five sequences (1, 127, 128, 300 and 1000 tokens, plus an empty one) packed along the token
    axis: each sequence's rows equal the oracle's forward over that sequence alone."""
    Hq, Hkv, d = 10, 2, 128
    pat = cw.Pattern(32, 200, 1000, 2)
    lens = [1, 127, 0, 128, 300, 1000]
    total = sum(lens)
    q64, q = host_and_device((1, total, Hq, d), "q", cuda_device, 29)
    k64, k = host_and_device((1, total, Hkv, d), "k", cuda_device, 29)
    v64, v = host_and_device((1, total, Hkv, d), "v", cuda_device, 29)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    o, lse = cw.cowa_fwd_varlen(q[0], k[0], v[0], torch.tensor(cu, device=cuda_device), pat)
    torch.cuda.synchronize()
    for s_, (a_, b_) in enumerate(zip(cu[:-1], cu[1:])):
        if b_ == a_:
            continue
        want_o, want_l = orc.attention_fwd(q64[:, a_:b_], k64[:, a_:b_], v64[:, a_:b_], oracle_pattern(pat))
        err_o = np.abs(to64(o[a_:b_]) - want_o[0]).max()
        err_l = np.abs(lse[:, a_:b_].cpu().numpy().astype(np.float64) - want_l[0]).max()
        assert err_o <= O_ATOL and err_l <= LSE_ATOL, (s_, err_o, err_l)
