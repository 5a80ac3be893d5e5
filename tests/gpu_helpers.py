"""Helpers shared by the GPU parity tests: input construction and tolerance checks.

Inputs are generated once (seeded, see structured_sparse_attention_cowa_b200.synth) and
handed to both sides: the CUDA path gets the bf16 device tensor, the oracle the same bits
widened exactly to float64.
"""

import numpy as np
import torch

from oracle import cowa_oracle as orc
from structured_sparse_attention_cowa_b200 import synth

O_ATOL = 2e-2    # output max-abs error vs fp64 (bf16 I/O)
LSE_ATOL = 1e-3  # lse max-abs error vs fp64
GRAD_RTOL = 1e-2  # relative Frobenius error of dq, dk, dv
# Relative error is undefined where the exact gradient is zero.  With one visible key per row (a
# sequence of length 1, or S = 0, L = 1 and no interval) P = 1 and dP = Delta, so dq = dk = 0 in
# exact arithmetic and the library's result is pure fp32 rounding.  A gradient whose fp64 norm is
# below VANISH times its cancellation-free bound B (see grad_bounds) counts as zero; its absolute
# Frobenius error must then stay below GRAD_RTOL * 2**-8 * B, one bf16 rounding of the terms the
# gradient is summed from.
VANISH = 1e-9


def host_and_device(shape, name, device, extra=0):
    """Seeded bf16 tensor: (float64 numpy copy for the oracle, bf16 CUDA tensor)."""
    bits = synth.normal_bf16_bits(shape, synth.seed_of(name, extra))
    return orc.bf16_bits_to_f64(bits), synth.bits_to_torch(bits, device)


class DeviceView:
    """Indexable like a numpy array; each index copies only that slice of a bf16 CUDA tensor
    to the host as float64 (exact widening), so the oracle can read multi-GB inputs."""

    def __init__(self, t):
        self.t = t
        self.shape = tuple(t.shape)

    def __getitem__(self, idx):
        idx = tuple(torch.as_tensor(i, device=self.t.device) if isinstance(i, np.ndarray) else i
                    for i in (idx if isinstance(idx, tuple) else (idx,)))
        return self.t[idx].float().cpu().numpy().astype(np.float64)


def to64(t):
    return t.float().cpu().numpy().astype(np.float64)


def oracle_pattern(p):
    return orc.Pattern(S=p.S, L=p.L, T=p.T, D=p.D, kv_head_base=p.kv_head_base,
                       h_kv_global=p.h_kv_global or None, scale=p.softmax_scale or None)


def rel_fro(a, b):
    """Relative Frobenius error ||a - b|| / ||b|| (b the fp64 reference, nonzero)."""
    nb = np.linalg.norm(b.ravel())
    assert nb > 0, "relative error of a vanishing reference: use grad_errors"
    return float(np.linalg.norm((a - b).ravel()) / nb)


def grad_bounds(q, k, v, do, scale):
    """Cancellation-free bounds on ||dq||, ||dk||, ||dv|| (Frobenius) of one attention call.

    Arrays [B, N, H, d] (float64).  Every softmax row sums to one and |dP_ts - Delta_t| <=
    2 ||dO_t|| max_s ||v_s|| (o_t is a convex combination of the v_s), so by the triangle
    inequality ||dq|| <= 2 scale max||k_s|| max||v_s|| ||dO||, and ||dk||, ||dv|| are bounded by
    the same terms with the sum of the rows' ||dO_t|| in place of ||dO||."""
    rn = lambda x: np.sqrt((x * x).sum(-1))
    mq, mk, mv = rn(q).max(), rn(k).max(), rn(v).max()
    l1 = rn(do).sum()
    return 2 * scale * mk * mv * np.linalg.norm(do), 2 * scale * mq * mv * l1, l1


def grad_errors(got, want, bounds):
    """Errors of (dq, dk, dv) in units of GRAD_RTOL's scale: relative Frobenius error, or for a
    vanishing reference the absolute error over 2**-8 times its bound (see VANISH)."""
    out = []
    for a, b, bound in zip(got, want, bounds):
        nb = float(np.linalg.norm(b.ravel()))
        den = nb if nb > VANISH * bound else 2.0 ** -8 * bound
        out.append(float(np.linalg.norm((a - b).ravel())) / den)
    return tuple(out)


def edge_rows(N, p, h_kv, extra_random=0, seed=0):
    """Rows at every pattern edge (sink, interval bounds, band width, ends) plus random rows."""
    H = p.h_kv_global or h_kv
    b = orc.interval_bounds(p.S, p.T, H)
    cand = {0, 1, p.S - 1, p.S, p.L - 1, p.L, N - 1, N - 2}
    for x in b:
        cand |= {x - 1, x, x + p.L - 1, x + p.L}
    rows = {r for r in cand if 0 <= r < N}
    rng = np.random.default_rng(seed)
    if extra_random:
        rows |= set(rng.integers(0, N, extra_random).tolist())
    return np.array(sorted(rows), dtype=np.int64)
