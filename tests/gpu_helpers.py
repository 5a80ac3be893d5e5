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
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-30))


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
