"""The FMA-pipe exp2 of the kernels: its constants are the ones the committed fit produces, and
its float32 evaluation (same steps as the device code) stays within the stated bound of
the true 2^x, computed in float64."""

import os
import re
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "structured_sparse_attention_cowa_b200", "csrc")
sys.path.insert(0, CSRC)

import exp2_poly_fit  # noqa: E402


def _header_coefs():
    txt = open(os.path.join(CSRC, "exp2_poly.cuh")).read()
    vals = {int(k): float(v) for k, v in re.findall(r"kExp2C(\d) = ([0-9.eE+-]+)f;", txt)}
    return np.array([vals[i] for i in range(4)], dtype=np.float32)


def test_header_matches_fit():
    c32 = exp2_poly_fit.fit().astype(np.float32)
    assert np.array_equal(_header_coefs(), c32)


def test_float32_evaluation_error_bound():
    c32 = _header_coefs()
    xs = np.concatenate([np.linspace(-120.0, 8.0, 400001), -np.logspace(-8, 2, 2001), [0.0, -1.0, 1.0, 8.0]])
    xs = xs.astype(np.float32)
    got = exp2_poly_fit.eval_f32(c32, xs).astype(np.float64)
    rel = np.abs(got / np.exp2(xs.astype(np.float64)) - 1.0)
    assert rel.max() < 8e-5
    # clamped below -120: a tiny positive normal float, never negative, denormal or NaN
    y = exp2_poly_fit.eval_f32(c32, np.array([-1000.0, -121.0], np.float32))
    assert (y > np.float32(2.0 ** -121)).all() and (y < np.float32(2.0 ** -119)).all()


def test_packed_variant_uses_the_same_steps():
    """The packed device variant repeats the scalar steps on pairs; its header text must carry
    the same constants and clamp (one source of truth: the kExp2C* constants)."""
    txt = open(os.path.join(CSRC, "exp2_poly.cuh")).read()
    body = txt[txt.index("exp2_fma_x2"):]
    for name in ("kExp2C3", "kExp2C2", "kExp2C1", "kExp2C0", "-120.0f", "12582912.0f"):
        assert name in body
