"""cowa_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers cannot allocate device memory on the serving path (runtimes that own the whole
memory pool, or code that must not call cudaMalloc because it synchronizes the device).  This
entry point keeps its split partials in the library's own static per-device scratch instead of
a caller workspace.  Checked through the C ABI against cowa_decode (which uses a caller
workspace) on two calls in a row with different inputs, within the decode tolerances of the
other parity tests; the second call must not see anything left over from the first.  That a
call allocates nothing is checked twice: torch's allocator count is unchanged, and the device's
free memory as the driver reports it (cudaMemGetInfo) does not drop across the second call (any
device allocation, however small, takes at least one 2 MiB page; the first call of a process may
load the library's device code, whose static scratch is part of that load).  The scratch's status word is read
back through cowa_decode_noalloc_status.  Also checks that a configuration too large for the
scratch is refused before any launch.  This file is collected last on purpose."""

import ctypes

import numpy as np
import pytest
import torch

from structured_sparse_attention_cowa_b200 import cowa as cw
from structured_sparse_attention_cowa_b200 import synth
from tests.gpu_helpers import LSE_ATOL, O_ATOL

pytestmark = pytest.mark.gpu


def _call_noalloc(pat, qt, kc, vc, pos, out, lse):
    B, Hq, d = qt.shape
    Hkv, T_cap = kc.shape[1], kc.shape[2]
    p = pat.c()
    return cw.lib().cowa_decode_noalloc(ctypes.byref(p), B, Hq, Hkv, d, T_cap, ctypes.c_void_p(qt.data_ptr()),
                                        cw._cache_tensor(kc, "bhtd"), cw._cache_tensor(vc, "bhtd"),
                                        ctypes.c_void_p(pos.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                        ctypes.c_void_p(lse.data_ptr()),
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_decode_matches_workspace_decode_twice(cuda_device):
    B, Hq, Hkv, d, T_cap = 4, 10, 2, 128, 3000
    pat = cw.Pattern(64, 256, 3000, 2)
    kc = synth.cuda_normal_bf16((B, Hkv, T_cap, d), synth.seed_of("k_cache", 11), cuda_device)
    vc = synth.cuda_normal_bf16((B, Hkv, T_cap, d), synth.seed_of("v_cache", 11), cuda_device)
    calls = [
        (synth.cuda_normal_bf16((B, Hq, d), synth.seed_of("q_t", 11), cuda_device), [2999, 0, 1500, 64]),
        (synth.cuda_normal_bf16((B, Hq, d), synth.seed_of("q_t", 12), cuda_device), [700, 2998, 63, 2000]),
    ]
    out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=cuda_device)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=cuda_device)
    for i, (qt, pos_list) in enumerate(calls):
        pos = torch.tensor(pos_list, dtype=torch.int32, device=cuda_device)
        want_o, want_l = cw.cowa_decode(qt, kc, vc, pos, pat)
        torch.cuda.synchronize()
        out.fill_(float("nan"))
        lse.fill_(float("nan"))
        before = torch.cuda.memory_allocated(cuda_device)
        free_before = torch.cuda.mem_get_info(cuda_device)[0]
        st = _call_noalloc(pat, qt, kc, vc, pos, out, lse)
        torch.cuda.synchronize()
        assert st == 0, cw.lib().cowa_status_string(st)
        assert torch.cuda.memory_allocated(cuda_device) == before
        if i > 0:  # the first call may load the library's device code, scratch included
            assert free_before - torch.cuda.mem_get_info(cuda_device)[0] < 2 * 1024 * 1024
        assert cw.decode_noalloc_status() == 0
        err_o = float((out.float() - want_o.float()).abs().max())
        err_l = float((lse - want_l).abs().max())
        assert np.isfinite(err_o) and np.isfinite(err_l)
        assert err_o <= O_ATOL and err_l <= LSE_ATOL, (pos_list, err_o, err_l)


def test_noalloc_decode_refuses_oversized_configuration(cuda_device):
    # a batch whose split partials need more than the scratch holds
    B, Hq, Hkv, d, T_cap = 64, 64, 8, 128, 131072
    pat = cw.Pattern(128, 4096, 131072, 8)
    need = cw.lib().cowa_decode_workspace_size(ctypes.byref(pat.c()), B, Hq, Hkv, d, T_cap)
    assert need > 8 * 1024 * 1024
    tiny = torch.zeros(16, dtype=torch.bfloat16, device=cuda_device)
    kc = torch.empty(0, dtype=torch.bfloat16, device=cuda_device)
    p = pat.c()
    t = cw.c_tensor(tiny.data_ptr(), 16, 16, 16)
    st = cw.lib().cowa_decode_noalloc(ctypes.byref(p), B, Hq, Hkv, d, T_cap, ctypes.c_void_p(tiny.data_ptr()), t, t,
                                      ctypes.c_void_p(tiny.data_ptr()), ctypes.c_void_p(tiny.data_ptr()), None,
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 4  # COWA_ERR_WORKSPACE, nothing launched
