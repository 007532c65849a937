"""The FMA-pipe exp2 of the tensor-core softmax (tc_util.cuh, exp2_poly2):
its polynomial for 2^f on [0, 1) must stay within the relative error that
the bf16 rounding of P hides.  The constants are read from the header and
the device algorithm (floor split, Horner, exponent add) is replayed in
float32 against float64 2^x."""

import os
import re

import numpy as np

HEADER = os.path.join(os.path.dirname(__file__), "..", "block_sparse_approximate_b200", "csrc", "tc_util.cuh")


def _coefficients():
    src = open(HEADER).read()
    m = re.search(r"constexpr float kC0 = ([0-9.eE+-]+)f, kC1 = ([0-9.eE+-]+)f, kC2 = ([0-9.eE+-]+)f, "
                  r"kC3 = ([0-9.eE+-]+)f;", src)
    assert m, "exp2_poly2 constants not found"
    return [np.float32(float(x)) for x in m.groups()]


def _exp2_poly(x):
    c0, c1, c2, c3 = _coefficients()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    n = np.floor(x)
    f = (x - n).astype(np.float32)
    q = (c3 * f + c2).astype(np.float32)
    q = (q * f + c1).astype(np.float32)
    q = (q * f + c0).astype(np.float32)
    return np.ldexp(q.astype(np.float64), n.astype(np.int64))


def test_relative_error_below_bf16_rounding():
    # the softmax feeds it x = s·(q·k) − m ≤ 2^8 (lazy rescale) down to the clamp
    x = np.linspace(-126.0, 8.0, 1_000_001, dtype=np.float64).astype(np.float32)
    rel = np.abs(_exp2_poly(x) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1e-4, rel.max()
    assert rel.max() < 2.0 ** -9 / 8      # well under the bf16 rounding of P


def test_integer_points_and_clamp():
    # f = 0: 2^n up to the constant term's error; below -126 the value stays tiny, not zero
    for n in (-20, -1, 0, 1, 7):
        v = _exp2_poly(np.array([n], dtype=np.float32))[0]
        assert abs(v / 2.0 ** n - 1.0) < 1e-4
    tiny = _exp2_poly(np.array([-1000.0, -np.inf], dtype=np.float32))
    assert np.all(tiny > 0) and np.all(tiny < 2.0 ** -125)
