"""The kernels' software exp2 (used for part of the softmax exponentials so
that the FMA pipe shares the MUFU's work), checked against fp64 exp2.

Method, as the kernels compute it (float32 throughout):
  x <- max(x, -125); t = x + 1.5*2^23 (round to nearest integer into the low
  mantissa bits); f = x - (t - 1.5*2^23) in [-1/2, 1/2]; p = Horner(f) with the
  coefficients of csrc/exp2_poly.h (a minimax-relative fit, fit_exp2_poly.py);
  result bits = bits(p) + (bits(t) << 23), i.e. p * 2^n.
"""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "ring_ulysses_sequence_b200", "csrc", "exp2_poly.h")


def coeffs():
    text = open(HDR).read()
    deg = int(re.search(r"RM_EXP2_POLY_DEG (\d+)", text).group(1))
    return [np.float32(float(re.search(rf"RM_EXP2_C{i} ([-0-9.e]+)f", text).group(1)))
            for i in range(deg + 1)]


def soft_exp2(x):
    c = coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    p = c[-1]
    for coef in c[-2::-1]:
        p = (p * f + coef).astype(np.float32)
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_over_the_softmax_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-125, 9, 2_000_001), rng.uniform(-30, 8, 1_000_000),
                        np.arange(-125, 9).astype(np.float64)]).astype(np.float32)
    y = soft_exp2(x).astype(np.float64)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(y - exact) / exact
    assert rel.max() < 2e-5, rel.max()          # the fit itself is ~5e-6
    assert np.all(np.isfinite(y))


def test_masked_inputs_go_to_zero():
    y = soft_exp2(np.array([-np.inf, -1e30, -200.0, -126.0], dtype=np.float32))
    assert np.all(y >= 0) and np.all(y <= 2.0 ** -124)


def test_fit_is_a_minimax_relative_polynomial():
    c = np.array(coeffs(), dtype=np.float64)
    assert c[0] == 1.0
    f = np.linspace(-0.5, 0.5, 100001)
    err = (np.polyval(c[::-1], f) - np.exp2(f)) / np.exp2(f)
    # equi-oscillation: the error reaches its bound with both signs several times
    bound = np.abs(err).max()
    assert bound < 1e-5
    assert (err > 0.9 * bound).any() and (err < -0.9 * bound).any()
