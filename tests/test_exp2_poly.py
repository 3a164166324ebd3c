"""CPU checks of the polynomial 2^x that the kernels run on the FP32 pipe.

The constants in csrc/sm100_ptx.cuh must be the ones the committed Remez fit
(causal_attention_fwd_b200/exp2_fit.py) produces, and the fp32 emulation of the
kernels' steps (clamp, magic-number rounding, Horner, exponent add) must stay
within the stated relative error against the exact 2^x on the whole input range
the softmax produces, with every input at or below the clamp giving 2^-126.
"""
import os
import re

import numpy as np

from causal_attention_fwd_b200 import exp2_fit

PTX = os.path.join(os.path.dirname(os.path.dirname(__file__)), "causal_attention_fwd_b200", "csrc",
                   "sm100_ptx.cuh")


def test_remez_fit_converged_to_equioscillation():
    c = exp2_fit.remez()
    f = np.linspace(-0.5, 0.5, 400001)
    e = exp2_fit._err(c, f)
    # a degree-3 minimax fit: 5 alternating extrema of equal size
    s = np.sign(e)
    segs = np.split(np.arange(f.size), np.flatnonzero(np.diff(s)) + 1)
    ext = np.array([np.abs(e[g]).max() for g in segs])
    assert len(segs) == 5
    assert ext.max() / ext.min() < 1.0 + 1e-6


def test_header_constants_are_the_fit():
    text = open(PTX).read()
    got = {int(k): np.float32(v) for k, v in re.findall(r"EXP2_C(\d) = ([0-9.e+-]+)f", text)}
    want = exp2_fit.fp32_coefficients()
    assert sorted(got) == [0, 1, 2, 3]
    for k in range(4):
        assert got[k] == want[k], (k, got[k], want[k])


def test_relative_error_bound_over_the_softmax_range():
    c = exp2_fit.fp32_coefficients()
    assert exp2_fit.max_rel_error(c) <= 7.5e-5
    x = np.linspace(-125.0, 64.0, 2000003).astype(np.float32)
    y = exp2_fit.exp2_emulated(x, c).astype(np.float64)
    rel = y / np.exp2(x.astype(np.float64)) - 1.0
    assert np.abs(rel).max() <= 7.5e-5
    assert abs(rel.mean()) <= 1e-5  # nearly unbiased: row sums (and LSE) are not shifted


def test_integers_and_halves():
    c = exp2_fit.fp32_coefficients()
    x = np.arange(-125, 40, 0.5).astype(np.float32)
    y = exp2_fit.exp2_emulated(x, c).astype(np.float64)
    np.testing.assert_allclose(y, np.exp2(x.astype(np.float64)), rtol=7.5e-5)


def test_clamp_gives_smallest_normal_not_garbage():
    c = exp2_fit.fp32_coefficients()
    x = np.array([-np.inf, -1e30, -1000.0, -200.0, -127.0, -126.0], np.float32)
    y = exp2_fit.exp2_emulated(x, c)
    assert np.all(np.isfinite(y)) and np.all(y > 0)
    assert np.all(np.abs(y.astype(np.float64) / 2.0**-126 - 1) <= 2e-4)
