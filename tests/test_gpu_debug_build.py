"""GPU: the self-checking build (libcowa_debug.so, COWA_DEBUG=1).

In that build every kernel checks each planned tile and cache row against the call's tensors
before its TMA load (a failed check reports COWA_ERR_CHECK through the workspace status and
skips the load; nothing traps).  On the awkward shapes below (ragged tails, GQA groups of 1 and
5, N > T, dense causal, d = 64, one KV head (split key tiles), a packed batch with empty and
length-1 sequences, a chunk of queries against a decode cache, full and compacted caches in bf16
and E4M3) no check fails and every output equals the release build's bit for bit."""

import pytest
import torch

from structured_sparse_attention_cowa_b200 import build as cbuild
from structured_sparse_attention_cowa_b200 import cowa as cw
from structured_sparse_attention_cowa_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def libs():
    release = cw.lib()
    path = cbuild.build(debug=True)
    saved_path = cw.LIB_PATH
    cw._lib, cw.LIB_PATH = None, path
    try:
        debug = cw.lib()
    finally:
        cw._lib, cw.LIB_PATH = release, saved_path
    return release, debug


def _both(libs, fn, device):
    """fn(ws) on the release and on the debug library; the debug run's status must be COWA_OK."""
    out = []
    for L in libs:
        ws = torch.zeros(64 << 20, dtype=torch.uint8, device=device)
        saved = cw._lib
        cw._lib = L
        try:
            r = fn(ws)
            torch.cuda.synchronize()
            assert cw.workspace_status(ws) == cw.COWA_OK
        finally:
            cw._lib = saved
        out.append([x.clone() for x in r])
    for a, b in zip(*out):
        assert torch.equal(a, b)


def _rand(shape, name, extra, device):
    return synth.cuda_normal_bf16(shape, synth.seed_of(name, extra), device)


@pytest.mark.parametrize("B,N,Hq,Hkv,d,pat", [
    (1, 1000, 10, 2, 128, cw.Pattern(64, 128, 1000, 2)),      # ragged tail, group of 5
    (2, 333, 4, 4, 128, cw.Pattern(5, 40, 333, 4)),           # group of 1, unaligned sink
    (1, 700, 8, 4, 128, cw.Pattern(32, 100, 500, 4)),         # N > T
    (1, 640, 8, 2, 128, cw.Pattern(16, 640, 640, 2)),         # dense causal
    (1, 300, 8, 4, 64, cw.Pattern(8, 32, 300, 2)),            # d = 64, duplicated windows
    (1, 4096, 4, 1, 128, cw.Pattern(64, 256, 4096, 1)),       # one KV head: long key tiles split
])
def test_debug_build_fwd_bwd(libs, cuda_device, B, N, Hq, Hkv, d, pat):
    q, k, v, do = (_rand(s, n, 21, cuda_device) for s, n in (((B, N, Hq, d), "q"), ((B, N, Hkv, d), "k"),
                                                               ((B, N, Hkv, d), "v"), ((B, N, Hq, d), "do")))

    def run(ws):
        o, lse = cw.cowa_fwd(q, k, v, pat, workspace=ws)
        dq, dk, dv = cw.cowa_bwd(q, k, v, o, lse, do, pat, workspace=ws)
        return o, lse, dq, dk, dv

    _both(libs, run, cuda_device)


def test_debug_build_packed_batch(libs, cuda_device):
    lens = [1, 127, 0, 128, 300, 1000]
    total, Hq, Hkv, d = sum(lens), 8, 2, 128
    pat = cw.Pattern(16, 64, 1024, 2)
    cu = torch.tensor([0] + list(torch.tensor(lens).cumsum(0)), dtype=torch.int32, device=cuda_device)
    q, k, v, do = (_rand(s, n, 22, cuda_device) for s, n in (((total, Hq, d), "q"), ((total, Hkv, d), "k"),
                                                               ((total, Hkv, d), "v"), ((total, Hq, d), "do")))

    def run(ws):
        o, lse = cw.cowa_fwd_varlen(q, k, v, cu, pat, workspace=ws)
        dq, dk, dv = cw.cowa_bwd_varlen(q, k, v, o, lse, do, cu, pat, workspace=ws)
        return o, lse, dq, dk, dv

    _both(libs, run, cuda_device)


def test_debug_build_chunk_and_decodes(libs, cuda_device):
    B, Hq, Hkv, d, Tc = 4, 8, 4, 128, 1024
    pat = cw.Pattern(32, 200, 1024, 4)
    kc = _rand((B, Hkv, Tc, d), "k_cache", 23, cuda_device)
    vc = _rand((B, Hkv, Tc, d), "v_cache", 23, cuda_device)
    qt = _rand((B, Hq, d), "q_t", 23, cuda_device)
    qb = _rand((B, 100, Hq, d), "q", 23, cuda_device)
    pos = torch.tensor([0, 63, 700, 1023], dtype=torch.int32, device=cuda_device)
    kc8, vc8 = cw.quantize_e4m3(kc, 1.0 / 64), cw.quantize_e4m3(vc, 1.0 / 64)
    kcc, vcc = cw.compact_cache(kc.transpose(1, 2), vc.transpose(1, 2), pat)
    kcc8, vcc8 = cw.compact_cache_fp8(kc8.transpose(1, 2).contiguous(), vc8.transpose(1, 2).contiguous(), pat)
    pos_c = torch.full((B,), Tc - 1, dtype=torch.int32, device=cuda_device)  # the compacted caches end there

    def run(ws):
        o1, l1 = cw.cowa_fwd_chunk(qb, kc, vc, pat, q_offset=900, kv_layout="bhtd", workspace=ws)
        o2, l2 = cw.cowa_decode(qt, kc, vc, pos, pat, workspace=ws)
        o3, l3 = cw.cowa_decode_compact(qt, kcc, vcc, pos_c, pat, workspace=ws)
        o4, l4 = cw.cowa_decode_fp8(qt, kc8, vc8, pos, pat, 1.0 / 64, 1.0 / 64, workspace=ws)
        o5, l5 = cw.cowa_decode_fp8_compact(qt, kcc8, vcc8, pos_c, pat, 1.0 / 64, 1.0 / 64, workspace=ws)
        return o1, l1, o2, l2, o3, l3, o4, l4, o5, l5

    _both(libs, run, cuda_device)
