"""GPU parity: cowa_bwd (through the C ABI) against the fp64 oracle.

Tolerance: relative Frobenius error <= 1e-2 for dq, dk, dv against fp64 gradients of
sum(dO * O) on identical bf16 inputs.  The forward output o and lse fed to the backward
come from cowa_fwd (as in training); the oracle recomputes everything from q, k, v, dO."""

import numpy as np
import pytest
import torch

from oracle import cowa_oracle as orc
from structured_sparse_attention_cowa_b200 import cowa as cw
from structured_sparse_attention_cowa_b200 import synth
from tests.gpu_helpers import (GRAD_RTOL, DeviceView, edge_rows, grad_bounds, grad_errors, host_and_device,
                               oracle_pattern, rel_fro, to64)

pytestmark = pytest.mark.gpu


def _inputs(B, N, Hq, Hkv, d, device, extra=0, cuda_gen=False):
    if cuda_gen:
        t = [synth.cuda_normal_bf16(s, synth.seed_of(n, extra), device)
             for s, n in (((B, N, Hq, d), "q"), ((B, N, Hkv, d), "k"), ((B, N, Hkv, d), "v"), ((B, N, Hq, d), "do"))]
        return [DeviceView(x) for x in t], t
    pairs = [host_and_device(s, n, device, extra)
             for s, n in (((B, N, Hq, d), "q"), ((B, N, Hkv, d), "k"), ((B, N, Hkv, d), "v"), ((B, N, Hq, d), "do"))]
    return [p[0] for p in pairs], [p[1] for p in pairs]


def _run(dev_inputs, pat):
    q, k, v, do = dev_inputs
    o, lse = cw.cowa_fwd(q, k, v, pat)
    dq, dk, dv = cw.cowa_bwd(q, k, v, o, lse, do, pat)
    torch.cuda.synchronize()
    return dq, dk, dv


def _check_full(B, N, Hq, Hkv, d, pat, device, extra=0):
    host, dev = _inputs(B, N, Hq, Hkv, d, device, extra)
    dq, dk, dv = _run(dev, pat)
    op = oracle_pattern(pat)
    want = orc.attention_bwd(*host, op)
    errs = grad_errors((to64(dq), to64(dk), to64(dv)), want, grad_bounds(*host, op.sm_scale(d)))
    assert max(errs) <= GRAD_RTOL, errs


def _unsplit_ws_bytes(B, N, Hq):
    n_pad = (N + 127) // 128 * 128
    return 256 + (2 * B * Hq * n_pad * 4 + 255) // 256 * 256


@pytest.mark.parametrize("B,N,Hq,Hkv,d,pat", [
    (1, 4096, 4, 1, 128, cw.Pattern(64, 256, 4096, 1)),     # one KV head: every key tile long
    (2, 3000, 2, 1, 64, cw.Pattern(16, 64, 3000, 1)),       # two sequences, ragged, d = 64
    (1, 4096, 4, 2, 128, cw.Pattern(32, 128, 4096, 2)),     # two KV heads: sink and interval tiles long
])
def test_bwd_split_key_tiles(cuda_device, B, N, Hq, Hkv, d, pat):
    """Calls with few KV heads cut the query range of their long key tiles into chunks run by
    CTAs of their own (fp32 partials summed in chunk order); the gradients match the oracle and
    two calls give the same bits."""
    import ctypes
    ws_bytes = cw.lib().cowa_bwd_workspace_size(ctypes.byref(pat.c()), B, N, Hq, Hkv, d)
    assert ws_bytes > _unsplit_ws_bytes(B, N, Hq)  # the plan splits this call
    host, dev = _inputs(B, N, Hq, Hkv, d, cuda_device, extra=17)
    q, k, v, do = dev
    o, lse = cw.cowa_fwd(q, k, v, pat)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=cuda_device)
    g1 = cw.cowa_bwd(q, k, v, o, lse, do, pat, workspace=ws)
    g2 = cw.cowa_bwd(q, k, v, o, lse, do, pat, workspace=ws)
    torch.cuda.synchronize()
    assert cw.workspace_status(ws) == 0
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)
    op = oracle_pattern(pat)
    want = orc.attention_bwd(*host, op)
    errs = grad_errors(tuple(to64(x) for x in g1), want, grad_bounds(*host, op.sm_scale(d)))
    assert max(errs) <= GRAD_RTOL, errs


def test_bwd_packed_qkv_layout(cuda_device):
    """The fused-projection layout of training: q, k, v as views into one packed
    [B, N, H_q + 2 H_kv, d] buffer, o and dO as views of wider buffers, and dq, dk, dv written
    into the matching views of one packed gradient buffer (nothing else of it touched).  The
    strided calls give the same bits as contiguous copies, and match the oracle."""
    B, N, Hq, Hkv, d = 2, 600, 8, 2, 128
    pat = cw.Pattern(32, 100, 600, 2)
    W = Hq + 2 * Hkv
    qkv64, qkv = host_and_device((B, N, W, d), "q", cuda_device, 13)
    do64, dobuf = host_and_device((B, N, 2 * Hq, d), "do", cuda_device, 13)
    q, k, v = qkv[:, :, :Hq], qkv[:, :, Hq:Hq + Hkv], qkv[:, :, Hq + Hkv:]
    do = dobuf[:, :, Hq:]
    obuf = torch.zeros((B, N, 2 * Hq, d), dtype=torch.bfloat16, device=cuda_device)
    o, lse = cw.cowa_fwd(q, k, v, pat, out=obuf[:, :, :Hq])
    gbuf = torch.full((B, N, W + 2, d), 7.0, dtype=torch.bfloat16, device=cuda_device)  # 2 spare heads
    dq, dk, dv = gbuf[:, :, :Hq], gbuf[:, :, Hq:Hq + Hkv], gbuf[:, :, Hq + Hkv:W]
    cw.cowa_bwd(q, k, v, o, lse, do, pat, dq=dq, dk=dk, dv=dv)
    qc, kc, vc, oc, doc = (x.contiguous() for x in (q, k, v, o, do))
    ref = cw.cowa_bwd(qc, kc, vc, oc, lse, doc, pat)
    torch.cuda.synchronize()
    for got, want in zip((dq, dk, dv), ref):
        assert torch.equal(got, want)
    assert bool((gbuf[:, :, W:] == 7.0).all())
    host = (qkv64[:, :, :Hq], qkv64[:, :, Hq:Hq + Hkv], qkv64[:, :, Hq + Hkv:], do64[:, :, Hq:])
    op = oracle_pattern(pat)
    want = orc.attention_bwd(*host, op)
    errs = grad_errors((to64(dq), to64(dk), to64(dv)), want, grad_bounds(*host, op.sm_scale(d)))
    assert max(errs) <= GRAD_RTOL, errs


def test_window_of_int_max_equals_dense_causal(cuda_device):
    """A band of L = INT_MAX (a caller's "no window limit") is the dense-causal mode: forward and
    backward give the same bits as L = N, and the gradients match the oracle.  The band ends
    s + L of the backward's row ranges must not overflow (they did before saturating)."""
    B, N, Hq, Hkv, d = 1, 700, 4, 2, 128
    host, dev = _inputs(B, N, Hq, Hkv, d, cuda_device, extra=11)
    wide, dense = cw.Pattern(16, 2**31 - 1, N, 2), cw.Pattern(16, N, N, 2)
    q, k, v, do = dev
    o1, l1 = cw.cowa_fwd(q, k, v, wide)
    o2, l2 = cw.cowa_fwd(q, k, v, dense)
    g1 = cw.cowa_bwd(q, k, v, o1, l1, do, wide)
    g2 = cw.cowa_bwd(q, k, v, o2, l2, do, dense)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)
    op = oracle_pattern(wide)
    want = orc.attention_bwd(*host, op)
    errs = grad_errors(tuple(to64(x) for x in g1), want, grad_bounds(*host, op.sm_scale(d)))
    assert max(errs) <= GRAD_RTOL, errs


@pytest.mark.parametrize("D", [4, 2, 1])
def test_bwd_tiny_config(cuda_device, D):
    """B=1, N=T=1024, H_q=8, H_kv=4, d=64, S=64, L=128; D=4 and the duplicated D=2, 1."""
    _check_full(1, 1024, 8, 4, 64, cw.Pattern(64, 128, 1024, D), cuda_device)


@pytest.mark.parametrize("B,N,Hq,Hkv,d,pat", [
    (1, 1000, 10, 2, 128, cw.Pattern(64, 128, 1000, 2)),     # ragged tail, group of 5
    (2, 333, 4, 4, 128, cw.Pattern(5, 40, 333, 4)),          # group of 1, unaligned sink
    (1, 77, 6, 2, 64, cw.Pattern(0, 1, 77, 2)),              # one partial tile, L = 1
    (1, 640, 8, 2, 128, cw.Pattern(16, 640, 640, 2)),        # dense causal
    (1, 520, 4, 2, 64, cw.Pattern(4, 60, 4, 1)),             # SWA + sinks
    (1, 700, 8, 4, 128, cw.Pattern(32, 100, 500, 4)),        # N > T
    (1, 300, 2, 1, 128, cw.Pattern(7, 30, 300, 2, kv_head_base=1, h_kv_global=2)),  # TP rank
    (1, 700, 8, 4, 128, cw.Pattern(16, 50, 2**31 - 1, 4)),   # declared span of INT_MAX: intervals past N
    (1, 300, 4, 2, 64, cw.Pattern(2**31 - 1, 1, 2**31 - 1, 2)),  # sink of INT_MAX: dense causal
    (1, 256, 16, 2, 64, cw.Pattern(16, 64, 256, 2, softmax_scale=0.3)),  # group of 8
    (2, 1, 10, 2, 128, cw.Pattern(64, 128, 1024, 2)),       # N = 1: one key per row, dq = dk = 0
    (1, 300, 8, 4, 128, cw.Pattern(0, 1, 0, 4)),            # S = 0, L = 1, T = 0: each row sees only itself
])
def test_bwd_edge_shapes(cuda_device, B, N, Hq, Hkv, d, pat):
    _check_full(B, N, Hq, Hkv, d, pat, cuda_device, extra=2)


def _check_sampled(B, N, Hq, Hkv, d, pat, device, rows, col_sets, cuda_gen):
    """dq on sampled rows (all heads) and dk/dv on sampled columns of some KV heads."""
    host, dev = _inputs(B, N, Hq, Hkv, d, device, cuda_gen=cuda_gen)
    dq, dk, dv = _run(dev, pat)
    op = oracle_pattern(pat)
    rows_t = torch.as_tensor(rows, device=device)
    wq = orc.attention_bwd_rows(*host, op, rows, b=0)
    assert rel_fro(to64(dq[0, rows_t]), wq) <= GRAD_RTOL
    for g, cols in col_sets:
        wk, wv = orc.attention_bwd_cols(*host, op, b=0, g=g, cols=cols)
        ct = torch.as_tensor(cols, device=device)
        assert rel_fro(to64(dk[0, ct, g]), wk) <= GRAD_RTOL, ("dk", g)
        assert rel_fro(to64(dv[0, ct, g]), wv) <= GRAD_RTOL, ("dv", g)
    # properties that hold at any size: softmax rows sum to one, and a shift of every key
    # by the same vector leaves the output unchanged
    grp = Hq // Hkv
    sum_dv = dv.double().sum(1)            # [B, Hkv, d]
    sum_do = dev[3].double().sum(1).view(B, Hkv, grp, d).sum(2)
    assert float((sum_dv - sum_do).norm() / sum_do.norm()) <= GRAD_RTOL
    sum_dk = dk.double().sum(1)
    assert float(sum_dk.norm() / dk.double().norm()) <= GRAD_RTOL
    return dq, dk, dv


def test_bwd_prefill_8k(cuda_device):
    """B=2, N=T=8192, H_q=32, H_kv=8, d=128, S=128, L=1024, D=8."""
    pat = cw.Pattern(128, 1024, 8192, 8)
    rows = edge_rows(8192, pat, 8, extra_random=128, seed=5)
    cols = [0, 127, 128, 129, 1100, 1151, 5000, 8191]
    _check_sampled(2, 8192, 32, 8, 128, pat, cuda_device, rows, [(0, cols), (7, cols)], cuda_gen=False)


def test_bwd_train_32k(cuda_device):
    """B=1, N=T=32768, H_q=40, H_kv=8, d=128, S=128, L=2048, D=8: sampled rows; for dk/dv the
    sink columns and the early-interval columns (the key tiles every later query tile visits:
    the longest accumulations), every interval edge of KV heads 0 and 1, band-only columns, the
    late interval of KV head 7 and the last key; and the any-size identities."""
    pat = cw.Pattern(128, 2048, 32768, 8)
    rows = edge_rows(32768, pat, 8, extra_random=96, seed=6)
    band_cols = [5000, 5001, 9000, 20000]
    sink = [0, 64, 127]
    head0 = [128, 129, 2000, 4207]        # interval [128, 4208) of KV head 0; 2000 is past the band of row 4100
    head1 = [4208, 4209, 8287]            # interval [4208, 8288) of KV head 1
    late = [28688, 28700, 30000, 32767]   # interval of KV head 7 and the last key
    _check_sampled(1, 32768, 40, 8, 128, pat, cuda_device, rows,
                   [(0, sink + head0 + band_cols), (1, sink[:1] + head1 + [9000]), (7, sink[:1] + band_cols + late)],
                   cuda_gen=True)


def test_bwd_long_128k(cuda_device):
    """B=1, N=T=131072, H_q=40, H_kv=8, d=128, S=128, L=4096, D=8: sampled rows; dk/dv at a sink
    column and the first interval column of KV head 0 (key tiles walked by all 1,024 query
    tiles), band-only columns, the last key; and the any-size identities."""
    pat = cw.Pattern(128, 4096, 131072, 8)
    rows = np.array([0, 127, 128, 4095, 4096, 16495, 16496, 70000, 131071])
    _check_sampled(1, 131072, 40, 8, 128, pat, cuda_device, rows,
                   [(0, [5, 128]), (3, [20000, 40001]), (7, [131071])], cuda_gen=True)


@pytest.mark.parametrize("B,N,Hq,Hkv,d,pat", [
    (1, 1500, 10, 2, 128, cw.Pattern(64, 200, 1500, 2)),
    (1, 4096, 4, 1, 128, cw.Pattern(64, 256, 4096, 1)),   # the dK/dV stage splits its key tiles
])
def test_bwd_stages_on_two_streams_match_single_call(cuda_device, B, N, Hq, Hkv, d, pat):
    """The staged entry point: preprocess, then dK/dV and dQ on two streams that both wait for
    it, gives the same bits as one cowa_bwd call (the kernels are deterministic)."""
    _, (q, k, v, do) = _inputs(B, N, Hq, Hkv, d, cuda_device, extra=9)
    o, lse = cw.cowa_fwd(q, k, v, pat)
    dq1, dk1, dv1 = cw.cowa_bwd(q, k, v, o, lse, do, pat)
    import ctypes
    n = cw.lib().cowa_bwd_workspace_size(ctypes.byref(pat.c()), B, N, Hq, Hkv, d)
    ws = torch.zeros(n, dtype=torch.uint8, device=cuda_device)
    dq2, dk2, dv2 = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    main = torch.cuda.current_stream()
    cw.cowa_bwd(q, k, v, o, lse, do, pat, dq=dq2, dk=dk2, dv=dv2, workspace=ws, stages=cw.BWD_PREPROCESS)
    ev = torch.cuda.Event()
    ev.record(main)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    s1.wait_event(ev)
    s2.wait_event(ev)
    cw.cowa_bwd(q, k, v, o, lse, do, pat, dq=dq2, dk=dk2, dv=dv2, workspace=ws, stages=cw.BWD_DKDV, stream=s1)
    cw.cowa_bwd(q, k, v, o, lse, do, pat, dq=dq2, dk=dk2, dv=dv2, workspace=ws, stages=cw.BWD_DQ, stream=s2)
    torch.cuda.synchronize()
    assert torch.equal(dq1, dq2) and torch.equal(dk1, dk2) and torch.equal(dv1, dv2)
