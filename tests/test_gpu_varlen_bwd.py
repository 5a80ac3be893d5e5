"""GPU parity: the backward of a packed variable-length batch (cowa_bwd_varlen: device cu_seqlens,
one launch per backward kernel over all sequences) against the fp64 oracle's backward over each
sequence alone.

Tolerance: relative Frobenius error <= 1e-2 for dq, dk, dv per sequence, as for cowa_bwd; the
length-1 sequence has dq = dk = 0 exactly and is judged by its absolute error (gpu_helpers.VANISH).
The o and lse fed to the backward come from cowa_fwd_varlen on the same packed batch.  Every
sequence is checked before the assertion, so a failure reports all of them."""

import numpy as np
import pytest
import torch

from oracle import cowa_oracle as orc
from structured_sparse_attention_cowa_b200 import cowa as cw
from tests.gpu_helpers import GRAD_RTOL, grad_bounds, grad_errors, host_and_device, oracle_pattern, to64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("Hq,Hkv,d,pat,lens", [
    (10, 2, 128, cw.Pattern(32, 200, 1000, 2), [1, 127, 0, 128, 300, 1000]),   # group of 5, an empty sequence
    (8, 4, 128, cw.Pattern(0, 40, 500, 4), [129, 257, 64]),                     # no sink, group of 2
    (4, 2, 64, cw.Pattern(8, 30, 200, 2), [int(x) for x in np.random.default_rng(3).integers(1, 150, 64)]),  # 64 short
    # one and two KV heads with long sequences: the long key tiles are split, planned on the device
    (4, 1, 128, cw.Pattern(64, 256, 4096, 1), [4096, 5, 1500, 0, 700]),
    (8, 2, 128, cw.Pattern(32, 128, 4096, 2), [3000, 1, 2000]),
])
def test_bwd_varlen_packed_batch(cuda_device, Hq, Hkv, d, pat, lens):
    total = sum(lens)
    q64, q = host_and_device((1, total, Hq, d), "q", cuda_device, 37)
    k64, k = host_and_device((1, total, Hkv, d), "k", cuda_device, 37)
    v64, v = host_and_device((1, total, Hkv, d), "v", cuda_device, 37)
    do64, do = host_and_device((1, total, Hq, d), "do", cuda_device, 37)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    cu_d = torch.tensor(cu, device=cuda_device)
    o, lse = cw.cowa_fwd_varlen(q[0], k[0], v[0], cu_d, pat)
    dq, dk, dv = cw.cowa_bwd_varlen(q[0], k[0], v[0], o, lse, do[0], cu_d, pat)
    torch.cuda.synchronize()
    op = oracle_pattern(pat)
    report = []
    for s_, (a_, b_) in enumerate(zip(cu[:-1], cu[1:])):
        if b_ == a_:
            continue
        sl = (q64[:, a_:b_], k64[:, a_:b_], v64[:, a_:b_], do64[:, a_:b_])
        want = [w[0] for w in orc.attention_bwd(*sl, op)]
        got = (to64(dq[a_:b_]), to64(dk[a_:b_]), to64(dv[a_:b_]))
        bounds = grad_bounds(*sl, op.sm_scale(d))
        report.append((s_, b_ - a_, grad_errors(got, want, bounds)))
    assert all(max(e) <= GRAD_RTOL for _, _, e in report), report
