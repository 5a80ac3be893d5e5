"""Pins of the oracle's E4M3 key/value format (oracle/fp8_kv.py) against things other than itself:
torch's float8_e4m3fn type (an independent library implementation of the OCP E4M3 format), the
format's landmark values worked out by hand from its definition, ties-to-even and saturation at
hand-computed midpoints, and the bf16 decode on caches whose values E4M3 holds exactly.  A few
plausible mistakes (wrong exponent bias, ties away from zero, no saturation, a dropped
subnormal range) are planted in copies here and must fail the same checks."""

import numpy as np
import pytest
import torch

from oracle import cowa_oracle as orc
from oracle import fp8_kv as f8

CODES = np.arange(256, dtype=np.uint8)


def _torch_values(codes):
    return torch.from_numpy(np.asarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def _torch_codes(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _same(a, b):
    return np.array_equal(np.isnan(a), np.isnan(b)) and np.array_equal(a[~np.isnan(a)], b[~np.isnan(b)])


def test_every_code_matches_torch():
    assert _same(f8.e4m3_to_f64(CODES), _torch_values(CODES))


@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6), (0x38, 1.0), (0x39, 1.125),
    (0x3F, 1.875), (0x40, 2.0), (0x77, 240.0), (0x7E, 448.0), (0xB8, -1.0), (0xFE, -448.0),
])
def test_landmark_values(code, value):
    """Subnormals m/8 * 2^-6, normals (1 + m/8) * 2^(e-7), largest finite 1.75 * 2^8 = 448."""
    assert f8.e4m3_to_f64([code])[0] == value


def test_nan_codes_and_negative_zero():
    v = f8.e4m3_to_f64([0x7F, 0xFF, 0x80])
    assert np.isnan(v[0]) and np.isnan(v[1]) and v[2] == 0.0 and np.signbit(v[2])
    assert f8.f64_to_e4m3([np.nan])[0] == 0x7F
    assert f8.f64_to_e4m3([-0.0])[0] == 0x80


def test_encode_decode_round_trip():
    fin = ~np.isnan(f8.e4m3_to_f64(CODES))
    assert np.array_equal(f8.f64_to_e4m3(f8.e4m3_to_f64(CODES[fin])), CODES[fin])


@pytest.mark.parametrize("x,code", [
    (1.0625, 0x38),             # midway 1.0 | 1.125: even mantissa 000
    (1.1875, 0x3A),             # midway 1.125 | 1.25: even mantissa 010
    (1.0625 + 1e-9, 0x39),      # just above the midpoint
    (2.0 ** -10, 0x00),         # midway 0 | 2^-9 (subnormal): even code 0
    (3 * 2.0 ** -10, 0x02),     # midway 2^-9 | 2^-8: even code 2
    (464.0, 0x7E),              # midway 448 | (480, not a value): saturates
    (1e6, 0x7E), (-1e6, 0xFE),  # saturation, sign kept
    (-1.1875, 0xBA),
])
def test_ties_to_even_and_saturation(x, code):
    assert f8.f64_to_e4m3([x])[0] == code


def test_rounding_matches_torch_in_range():
    """torch converts float32 to float8_e4m3fn with round-to-nearest-even; it agrees with the
    oracle wherever it does not overflow (|x| <= 464: above that torch gives NaN, the oracle
    saturates, which is the satfinite conversion's rule)."""
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.standard_normal(200000) * s for s in (1e-3, 0.05, 1.0, 30.0, 150.0)]).astype(np.float32)
    x = x[np.abs(x) <= 464]
    assert np.array_equal(f8.f64_to_e4m3(x.astype(np.float64)), _torch_codes(x))


def test_quantize_uses_a_float32_reciprocal():
    x = np.array([1.0, 3.0, -7.5, 150.0], dtype=np.float32)  # x / scale stays below 464
    scale = 0.37
    inv = np.float32(1.0) / np.float32(scale)
    assert np.array_equal(f8.quantize_e4m3_f32(x, scale), _torch_codes(x * inv))


def test_decode_fp8_equals_bf16_decode_on_exact_caches():
    """Cache values that E4M3 holds exactly (random codes; scales (1, 1) and (0.5, 2)): the FP8 decode is the
    bf16 decode of the same values (and scaling the cache scales the values it sees)."""
    rng = np.random.default_rng(3)
    B, Hq, Hkv, T_cap, d = 2, 4, 2, 300, 16
    pat = orc.Pattern(S=8, L=20, T=300, D=2)
    codes = lambda: f8.f64_to_e4m3(rng.standard_normal((B, Hkv, T_cap, d)))
    kc, vc = codes(), codes()
    qt = rng.standard_normal((B, Hq, d))
    pos = [299, 57]
    for ks, vs in ((1.0, 1.0), (0.5, 2.0)):
        o, lse = f8.decode_fp8(qt, kc, vc, ks, vs, pos, pat)
        wo, wl = orc.decode(qt, ks * f8.e4m3_to_f64(kc), vs * f8.e4m3_to_f64(vc), pos, pat)
        assert np.array_equal(o, wo) and np.array_equal(lse, wl)
    # scale by a power of two on the values: the output scales exactly
    o1, _ = f8.decode_fp8(qt, kc, vc, 1.0, 1.0, pos, pat)
    o2, _ = f8.decode_fp8(qt, kc, vc, 1.0, 4.0, pos, pat)
    assert np.allclose(o2, 4.0 * o1, rtol=0, atol=1e-12)


# ------------------------------------------------------------------ planted mistakes must fail
def _bias8(codes):
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    e, m = (c >> 3) & 0xF, c & 0x7
    v = np.where(e == 0, m / 8.0 * 2.0 ** -7, (1.0 + m / 8.0) * np.exp2(e - 8.0))
    return np.where((c & 0x7F) == 0x7F, np.nan, np.where(c & 0x80, -v, v))


def _no_subnormals(codes):
    v = f8.e4m3_to_f64(codes)
    c = np.asarray(codes, dtype=np.uint8)
    return np.where(((c >> 3) & 0xF) == 0, 0.0, v)


def _ties_away(x):
    out = f8.f64_to_e4m3(x)
    grid = f8.e4m3_to_f64(np.arange(0x7F, dtype=np.uint8))
    a = np.abs(np.asarray(x, dtype=np.float64))
    mid = (grid[:-1] + grid[1:]) / 2
    for i, ai in enumerate(a):
        k = np.nonzero(mid == ai)[0]
        if len(k):
            out[i] = (out[i] & 0x80) | (k[0] + 1)
    return out


def _no_saturation(x):
    out = f8.f64_to_e4m3(x)
    return np.where(np.abs(np.asarray(x)) > 464, np.uint8(0x7F), out).astype(np.uint8)


def test_planted_mistakes_are_caught():
    assert not _same(_bias8(CODES), _torch_values(CODES))
    assert not _same(_no_subnormals(CODES), _torch_values(CODES))
    assert _ties_away([1.0625])[0] != 0x38
    assert _no_saturation([1e6])[0] != 0x7E
