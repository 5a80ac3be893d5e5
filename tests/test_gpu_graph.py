"""GPU: the entry points are stream-ordered, allocate nothing and never synchronise the host, so a
training or serving step can be captured in a CUDA graph and replayed.  A forward + backward +
decode step (and a backward that splits its long key tiles) captured on a side stream and
replayed twice gives the same bits as the eager calls."""

import ctypes

import pytest
import torch

from structured_sparse_attention_cowa_b200 import cowa as cw
from structured_sparse_attention_cowa_b200 import synth

pytestmark = pytest.mark.gpu


def _rand(shape, name, dev):
    return synth.cuda_normal_bf16(shape, synth.seed_of(name, 51), dev)


@pytest.mark.parametrize("Hq,Hkv,N,pat", [
    (8, 2, 1500, cw.Pattern(32, 200, 1500, 2)),     # GQA layer, no split
    (4, 1, 4096, cw.Pattern(64, 256, 4096, 1)),     # one KV head: the backward splits its key tiles
])
def test_step_replays_from_a_cuda_graph(cuda_device, Hq, Hkv, N, pat):
    B, d, Tc = 1, 128, 2048
    q, k, v, do = (_rand(s, n, cuda_device) for s, n in (((B, N, Hq, d), "q"), ((B, N, Hkv, d), "k"),
                                                         ((B, N, Hkv, d), "v"), ((B, N, Hq, d), "do")))
    kc, vc = _rand((4, Hkv, Tc, d), "k_cache", cuda_device), _rand((4, Hkv, Tc, d), "v_cache", cuda_device)
    qt = _rand((4, Hq, d), "q_t", cuda_device)
    pos = torch.tensor([0, 100, 1500, Tc - 1], dtype=torch.int32, device=cuda_device)
    L, cp = cw.lib(), pat.c()
    ws = lambda n: torch.zeros(max(256, n), dtype=torch.uint8, device=cuda_device)
    ws_f = ws(L.cowa_fwd_workspace_size(ctypes.byref(cp), B, N, Hq, Hkv, d))
    ws_b = ws(L.cowa_bwd_workspace_size(ctypes.byref(cp), B, N, Hq, Hkv, d))
    ws_d = ws(L.cowa_decode_workspace_size(ctypes.byref(cp), 4, Hq, Hkv, d, Tc))
    o, lse = torch.empty_like(q), torch.empty((B, Hq, N), dtype=torch.float32, device=cuda_device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    od, lsed = torch.empty((4, Hq, d), dtype=torch.bfloat16, device=cuda_device), \
        torch.empty((4, Hq), dtype=torch.float32, device=cuda_device)
    outs = (o, lse, dq, dk, dv, od, lsed)

    def step(stream=None):
        cw.cowa_fwd(q, k, v, pat, out=o, lse=lse, workspace=ws_f, stream=stream)
        cw.cowa_bwd(q, k, v, o, lse, do, pat, dq=dq, dk=dk, dv=dv, workspace=ws_b, stream=stream)
        cw.cowa_decode(qt, kc, vc, pos, pat, out=od, lse=lsed, workspace=ws_d, stream=stream)

    step()
    torch.cuda.synchronize()
    want = [x.clone() for x in outs]
    for x in outs:
        x.zero_()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            step(stream=side)
    for _ in range(2):
        for x in outs:
            x.zero_()
        g.replay()
        torch.cuda.synchronize()
        for got, w in zip(outs, want):
            assert torch.equal(got, w)
    for w_ in (ws_f, ws_b, ws_d):
        assert cw.workspace_status(w_) == 0
    del g
