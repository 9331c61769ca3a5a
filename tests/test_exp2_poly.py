"""The FMA-pipe exponential of the attention softmax: its polynomial.

The kernels evaluate 2^x as 2^round(x) * p(f), f = x - round(x) in [-1/2, 1/2],
with p a degree-3 polynomial whose coefficients sit in csrc/common.cuh.  These
CPU tests read those four numbers from the source and pin them to the
mathematics: the relative error of p against numpy's exp2 over the whole
interval stays within the 7.5e-5 the kernels' documentation states (well under
the 2^-9 rounding of the bf16 P that follows), the error equioscillates as a
minimax fit does, and the reconstruction 2^n * p(f) covers the softmax's range.
"""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "block_sparse_attention_pool_b200", "csrc", "common.cuh")


def coefficients():
    text = open(SRC).read()
    c = [float(re.search(rf"constexpr float kExp2C{i} = ([0-9.eE+-]+)f;", text).group(1)) for i in range(4)]
    return np.array(c, dtype=np.float32).astype(np.float64)


def poly(c, f):
    return ((c[3] * f + c[2]) * f + c[1]) * f + c[0]


def test_relative_error_within_stated_bound():
    c = coefficients()
    f = np.linspace(-0.5, 0.5, 400_001)
    rel = poly(c, f) / np.exp2(f) - 1.0
    assert np.abs(rel).max() <= 7.5e-5
    # far below the bf16 rounding of P (half an ulp: 2^-9 relative)
    assert np.abs(rel).max() < 2.0 ** -13


def test_error_equioscillates_like_a_minimax_fit():
    c = coefficients()
    f = np.linspace(-0.5, 0.5, 400_001)
    rel = poly(c, f) / np.exp2(f) - 1.0
    # a degree-3 minimax fit has 5 alternating extrema of (nearly) equal size
    sign_changes = np.count_nonzero(np.diff(np.sign(rel[np.abs(rel) > 1e-7])))
    assert sign_changes == 4
    ends = np.abs([rel[0], rel[-1]])
    assert ends.min() > 0.9 * np.abs(rel).max()


def test_reconstruction_over_the_softmax_range():
    # x in [-125, 8]: n = round(x) in [-125, 8], p(f) in [2^-1/2, 2^1/2] (up to
    # the fit error), so 2^n p(f) is a normal fp32 number and the exponent add
    # of the kernels is exact
    c = coefficients()
    x = np.linspace(-125.0, 8.0, 200_001)
    n = np.rint(x)
    f = x - n
    y = np.ldexp(poly(c, f), n.astype(int))
    assert np.all(np.abs(f) <= 0.5)
    assert np.all(y >= np.finfo(np.float32).tiny)
    rel = y / np.exp2(x) - 1.0
    assert np.abs(rel).max() <= 7.5e-5
