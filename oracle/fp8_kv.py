"""FP8 (E4M3) key/value cache for CoWA decoding: the plain CPU definition.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference legs may import or call anything in this package; it
imports nothing from the library.

What it computes
----------------
The CoWA pages fix the attention pattern, not the storage precision of a decode cache.  An
8-bit cache halves the bytes a decode step reads (decode reads only the visible K/V rows and is
bound by memory bandwidth).  The format is E4M3 as the OCP 8-bit floating point specification
defines it (the "E4M3FN" variant: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, no
infinities, S.1111.111 is NaN, largest finite magnitude 448, subnormals m/8 * 2^-6).

Readings (this library's choices, the pages being silent):

* one scale per cache tensor: the stored key is ``e4m3(k / k_scale)`` and the attention uses
  ``k_scale * e4m3_value``, likewise for values with ``v_scale``;
* quantisation rounds to nearest, ties to even, and saturates: finite magnitudes beyond 448
  become 448 with their sign (the ``satfinite`` conversion); NaN stays NaN;
* the query stays in bf16; decoding over the FP8 cache is ``cowa_oracle.decode`` over the
  dequantised cache, so the only difference from the bf16 decode is the cache's rounding.

Pins (tests/test_oracle_fp8.py): all 256 codes against torch's ``float8_e4m3fn``; the spec's
landmark values; encode(decode(c)) == c for every finite code; ties to even and saturation at
hand-computed points; torch's own RNE conversion on random in-range values; the scaled decode
against the bf16 decode on caches whose values are exactly representable in E4M3.
"""

from __future__ import annotations

import numpy as np

from . import cowa_oracle as orc

__all__ = ["E4M3_MAX", "e4m3_to_f64", "f64_to_e4m3", "quantize_e4m3_f32", "decode_fp8"]

E4M3_MAX = 448.0


def e4m3_to_f64(codes) -> np.ndarray:
    """Value of each E4M3 code (uint8 array) as float64; NaN for the two NaN codes."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = sign * val
    return np.where((c & 0x7F) == 0x7F, np.nan, val)


def f64_to_e4m3(x) -> np.ndarray:
    """E4M3 code of each value: round to nearest, ties to even, saturating at +-448."""
    x = np.asarray(x, dtype=np.float64)
    nan = np.isnan(x)
    sgn = np.where(np.signbit(x) & ~nan, 0x80, 0x00)
    a = np.minimum(np.abs(np.where(nan, 0.0, x)), E4M3_MAX)
    # the 127 non-negative finite values in increasing code order (codes 0x00 .. 0x7E)
    grid = e4m3_to_f64(np.arange(0x7F, dtype=np.uint8))
    hi = np.searchsorted(grid, a, side="left")          # first grid value >= a
    lo = np.maximum(hi - 1, 0)
    dlo, dhi = a - grid[lo], grid[hi] - a
    exact = (hi == 0) | (grid[hi] == a)
    tie_pick = np.where(lo % 2 == 0, lo, hi)            # the code with an even mantissa
    code = np.where(exact, hi, np.where(dlo < dhi, lo, np.where(dhi < dlo, hi, tie_pick)))
    out = (sgn | code).astype(np.uint8)
    return np.where(nan, np.uint8(0x7F), out).astype(np.uint8)


def quantize_e4m3_f32(x, scale: float) -> np.ndarray:
    """Codes of ``x / scale`` the way a float32 kernel forms them: the reciprocal of the scale
    rounded to float32, one float32 multiply, then round-to-nearest-even saturating E4M3."""
    inv = np.float32(1.0) / np.float32(scale)
    y = np.asarray(x, dtype=np.float32) * inv
    return f64_to_e4m3(y.astype(np.float64))


def decode_fp8(q_t, k_codes, v_codes, k_scale: float, v_scale: float, pos, pat: orc.Pattern):
    """o[B,Hq,d], lse[B,Hq] of one new token per sequence over an E4M3 cache
    ([B, H_kv, T_cap, d] codes): the CoWA decode over k_scale * e4m3(k), v_scale * e4m3(v)."""
    k = k_scale * e4m3_to_f64(k_codes)
    v = v_scale * e4m3_to_f64(v_codes)
    return orc.decode(q_t, k, v, pos, pat)
