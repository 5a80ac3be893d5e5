"""GPU parity: decoding over an E4M3 (8-bit float) K/V cache against the fp64 oracle of that cache
(oracle/fp8_kv.py), and the quantiser that writes such a cache, bit for bit.

The E4M3 cache is this library's reading of the lower-memory decode cache next to the SWA
baseline ("Sliding Window Attention Beats Linear Attention ...", "Engineering Advantages"); the
pages fix no cache precision.  Tolerances are those of the bf16 decode (output max-abs 2e-2, lse
max-abs 1e-3 against fp64 over the same dequantised cache); the quantiser is integer work and is
compared exactly."""

import ctypes

import numpy as np
import pytest
import torch

from oracle import cowa_oracle as orc
from oracle import fp8_kv as f8
from structured_sparse_attention_cowa_b200 import cowa as cw
from structured_sparse_attention_cowa_b200 import synth
from tests.gpu_helpers import LSE_ATOL, O_ATOL, oracle_pattern

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("scale", [1.0, 0.37, 0.01])
def test_quantize_matches_oracle_bit_exact(cuda_device, scale):
    bits = synth.normal_bf16_bits((4096 * 8,), 77)
    x = orc.bf16_bits_to_f64(bits) * 20.0                       # well past 448 * scale: saturation
    x[:6] = [0.0, -0.0, 1e-30, -1e-30, 448.0 * scale, -464.0 * scale]  # zeros, underflow, the max, a tie
    bits = synth.f32_to_bf16_bits(x.astype(np.float32))
    got = cw.quantize_e4m3(synth.bits_to_torch(bits, cuda_device), scale).cpu().numpy()
    want = f8.quantize_e4m3_f32(orc.bf16_bits_to_f64(bits).astype(np.float32), scale)
    assert np.array_equal(got, want), np.flatnonzero(got != want)[:10]


def _codes(shape, seed, scale=3.0):
    return f8.f64_to_e4m3(np.random.default_rng(seed).standard_normal(shape) * scale)


@pytest.mark.parametrize("Hq,Hkv,pat,pos,layout", [
    (8, 4, cw.Pattern(64, 128, 1024, 4), [0, 63, 64, 200, 1023, 511], "bhtd"),
    (10, 2, cw.Pattern(20, 100, 900, 2), [899, 17, 1000, 5], "bhtd"),       # pos past T, group of 5
    (8, 8, cw.Pattern(0, 1, 1024, 8), [1023, 0, 700], "bthd"),             # no sink, L = 1, token-major
    (16, 2, cw.Pattern(4, 60, 4, 1), [1023, 3, 64], "bhtd"),               # SWA + sinks, group of 8
])
def test_decode_fp8_matches_oracle(cuda_device, Hq, Hkv, pat, pos, layout):
    B, d, T_cap = len(pos), 128, 1024
    kc, vc = _codes((B, Hkv, T_cap, d), 5), _codes((B, Hkv, T_cap, d), 6)
    qbits = synth.normal_bf16_bits((B, Hq, d), 9)
    ks, vs = 0.4, 0.25
    to_dev = (lambda c: torch.from_numpy(c).to(cuda_device)) if layout == "bhtd" else \
        (lambda c: torch.from_numpy(np.ascontiguousarray(c.transpose(0, 2, 1, 3))).to(cuda_device))
    n_ws = cw.lib().cowa_decode_fp8_workspace_size(ctypes.byref(pat.c()), B, Hq, Hkv, d, T_cap)
    ws = torch.zeros(max(256, n_ws), dtype=torch.uint8, device=cuda_device)
    o, lse = cw.cowa_decode_fp8(synth.bits_to_torch(qbits, cuda_device), to_dev(kc), to_dev(vc),
                                torch.tensor(pos, dtype=torch.int32, device=cuda_device), pat, ks, vs,
                                layout=layout, workspace=ws)
    assert cw.workspace_status(ws) == 0
    want_o, want_l = f8.decode_fp8(orc.bf16_bits_to_f64(qbits), kc, vc, ks, vs, pos, oracle_pattern(pat))
    assert np.abs(o.float().cpu().numpy() - want_o).max() <= O_ATOL
    assert np.abs(lse.cpu().numpy() - want_l).max() <= LSE_ATOL


def test_decode_fp8_compact_build_and_append_match_oracle(cuda_device):
    """Compacted E4M3 cache built from a prefill of N tokens, then tokens appended one at a time
    across the band ring's wrap; each decode against the oracle over the full code cache."""
    B, Hq, Hkv, d, N, T = 2, 8, 2, 128, 700, 1200
    pat = cw.Pattern(20, 100, T, 2)
    total = N + 160
    k8, v8 = _codes((B, total, Hkv, d), 11), _codes((B, total, Hkv, d), 12)   # [B, T, H_kv, d]
    kd, vd = torch.from_numpy(k8).to(cuda_device), torch.from_numpy(v8).to(cuda_device)
    kc, vc = cw.compact_cache_fp8(kd[:, :N].contiguous(), vd[:, :N].contiguous(), pat)
    kf, vf = np.ascontiguousarray(k8.transpose(0, 2, 1, 3)), np.ascontiguousarray(v8.transpose(0, 2, 1, 3))
    op = oracle_pattern(pat)
    for step, p in enumerate(range(N, total)):
        pos = torch.tensor([p, p], dtype=torch.int32, device=cuda_device)
        cw.compact_append_fp8(kc, vc, kd[:, p], vd[:, p], pos, pat)
        if step % 40 != 39:
            continue
        qbits = synth.normal_bf16_bits((B, Hq, d), 100 + step)
        o, lse = cw.cowa_decode_fp8_compact(synth.bits_to_torch(qbits, cuda_device), kc, vc, pos, pat, 0.5, 0.75)
        want_o, want_l = f8.decode_fp8(orc.bf16_bits_to_f64(qbits), kf, vf, 0.5, 0.75, [p, p], op)
        assert np.abs(o.float().cpu().numpy() - want_o).max() <= O_ATOL, p
        assert np.abs(lse.cpu().numpy() - want_l).max() <= LSE_ATOL, p


def test_decode_fp8_128k_config(cuda_device):
    """B=16, 131072-token cache quantised on the device from bf16 N(0,1) values (scale 1/64: the
    largest |x| of 8.6 G normals stays well below 448/64), H_q=40, H_kv=8, d=128, S=128, L=4096,
    D=8; the quantiser is checked bit-exact on a slice, the decode on sampled sequences."""
    B, Hq, Hkv, d, T_cap = 16, 40, 8, 128, 131072
    pat = cw.Pattern(128, 4096, 131072, 8)
    pos = [131071] * B
    pos[3], pos[5] = 70000, 4000
    scale = 1.0 / 64
    codes = []
    for name in ("k_cache", "v_cache"):
        x = synth.cuda_normal_bf16((B, Hkv, T_cap, d), synth.seed_of(name, 21), cuda_device)
        c = cw.quantize_e4m3(x, scale)
        xs = x[3, 2, 60000:64096].contiguous()
        want = f8.quantize_e4m3_f32(orc.bf16_bits_to_f64(synth.torch_to_bits(xs)).astype(np.float32), scale)
        assert np.array_equal(c[3, 2, 60000:64096].cpu().numpy(), want), name
        del x
        codes.append(c)
    qbits = synth.normal_bf16_bits((B, Hq, d), synth.seed_of("q_t", 21))
    o, lse = cw.cowa_decode_fp8(synth.bits_to_torch(qbits, cuda_device), codes[0], codes[1],
                                torch.tensor(pos, dtype=torch.int32, device=cuda_device), pat, scale, scale)
    torch.cuda.synchronize()
    q64 = orc.bf16_bits_to_f64(qbits)
    for b in (0, 3, 5):
        want_o, want_l = f8.decode_fp8(q64[b:b + 1], codes[0][b:b + 1].cpu().numpy(), codes[1][b:b + 1].cpu().numpy(),
                                       scale, scale, [pos[b]], oracle_pattern(pat))
        assert np.abs(o[b:b + 1].float().cpu().numpy() - want_o).max() <= O_ATOL, b
        assert np.abs(lse[b:b + 1].cpu().numpy() - want_l).max() <= LSE_ATOL, b
