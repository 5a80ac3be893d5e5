"""Plant plausible mistakes in the oracle (CPU only) and check that some pin catches each.

Each mutant replaces one oracle function with a subtly wrong copy (an
off-by-one band edge, a wrong interval slot, ceil instead of floor bounds, a
missing softmax scale in dk, a dropped max term in the lse) and runs the pins
that should fail on it.
"""

import numpy as np
import pytest

from oracle import cowa_oracle as orc
from tests import test_oracle_pins as pins


def _mask_band_off_by_one(rows, ncols, pat, g, h_kv):
    t = np.asarray(rows, dtype=np.int64)[:, None]
    s = np.arange(ncols, dtype=np.int64)[None, :]
    lo, hi = orc.interval_of(pat.kv_head_base + g, pat, h_kv)
    return (s <= t) & ((s < pat.S) | (s >= t - pat.L) | ((s >= lo) & (s < hi)))


def _interval_wrong_slot(G, pat, h_kv):
    H = pat.H(h_kv)
    b = orc.interval_bounds(pat.S, pat.T, H)
    p = G % H  # ignores D: every head gets its own window even in the duplicated ablation
    return b[p], b[p + 1]


def _bounds_ceil(S, T, H):
    R = T - S
    return [S + -((-i * R) // H) for i in range(H + 1)]


def _interval_local_index(G, pat, h_kv):
    # ignores the global head offset: uses the local index on every rank
    H = pat.H(h_kv)
    b = orc.interval_bounds(pat.S, pat.T, H)
    p = ((G - pat.kv_head_base) % pat.D) * (H // pat.D)
    return b[p], b[p + 1]


def _fwd_lse_without_max(q, k, v, pat):
    o, lse = orc_fwd_orig(q, k, v, pat)
    return o, lse - 0.5  # a dropped/shifted term in the lse


orc_fwd_orig = orc.attention_fwd
orc_bwd_orig = orc.attention_bwd


def _bwd_missing_scale(q, k, v, do, pat):
    dq, dk, dv = orc_bwd_orig(q, k, v, do, pat)
    d = np.asarray(q).shape[-1]
    return dq, dk / pat.sm_scale(d), dv


def _bwd_dv_transposed_heads(q, k, v, do, pat):
    dq, dk, dv = orc_bwd_orig(q, k, v, do, pat)
    return dq, dk, dv[:, :, ::-1].copy()


def _widen_shift_15(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 15).view(np.float32).astype(np.float64)


def _widen_sign_lost(bits):
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) & 0x7FFF
    return (b << 16).view(np.float32).astype(np.float64)


MUTANTS = [
    ("bf16_bits_to_f64", _widen_shift_15, [lambda: pins.test_bf16_widening_every_bit_pattern()]),
    ("bf16_bits_to_f64", _widen_sign_lost, [lambda: pins.test_bf16_widening_every_bit_pattern()]),
    ("visible_mask", _mask_band_off_by_one, [lambda: pins.test_visible_counts_brute_force_and_closed_form(120, 5, 9, 120, 4, 4),
                                            lambda: pins.test_swa_with_sinks_golden()]),
    ("interval_of", _interval_wrong_slot, [lambda: pins.test_ablation_distinct_windows_fixed_width()]),
    ("interval_bounds", _bounds_ceil, [lambda: pins.test_visible_counts_brute_force_and_closed_form(120, 5, 9, 120, 4, 4)]),
    ("interval_of", _interval_local_index, [lambda: pins.test_global_head_index_keeps_complementary_windows()]),
    ("attention_fwd", _fwd_lse_without_max, [lambda: pins.test_first_row_and_constant_values(),
                                              lambda: pins.test_dense_causal_special_case_matches_library_attention()]),
    ("attention_bwd", _bwd_missing_scale, [lambda: pins.test_bwd_central_finite_differences(2, 3, 16, 2)]),
    ("attention_bwd", _bwd_dv_transposed_heads, [lambda: pins.test_bwd_row_and_column_sum_identities()]),
]


@pytest.mark.parametrize("idx", range(len(MUTANTS)))
def test_pins_catch_planted_mistake(idx, monkeypatch):
    name, fn, checks = MUTANTS[idx]
    monkeypatch.setattr(orc, name, fn)
    for check in checks:
        with pytest.raises(AssertionError):
            check()
