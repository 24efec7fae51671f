"""Error bound of the cubic 2^x the forward kernel evaluates on the FMA pipe.

The coefficients are read from the CUDA header and the same float32 steps
(round-to-nearest split x = n + f, Horner cubic, exponent add) are replayed
with numpy; the result must stay within 1.1e-4 relative of 2^x, i.e. well below
the bf16 resolution (2^-9) the attention probabilities are rounded to."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "hierarchical_sparse_long_b200", "csrc", "tc_ptx.cuh")


def _coeffs():
    text = open(HDR).read()
    return [np.float32(1.0)] + [np.float32(float(re.search(rf"kExp2C{i} = ([0-9.eE+-]+)f;", text).group(1)))
                                for i in range(1, 4)]


def _ex2_poly(x):
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-125))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = ((c3 * f + c2).astype(np.float32) * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_ex2_poly_relative_error():
    x = np.linspace(-100.0, 8.0, 2_000_001).astype(np.float32)
    got = _ex2_poly(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 1.1e-4, rel.max()


def test_ex2_poly_exact_at_integers_and_clamped_below():
    x = np.arange(-125, 9, dtype=np.float32)  # results stay normal floats
    rel = np.abs(_ex2_poly(x).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() < 1.1e-4
    low = _ex2_poly(np.array([-1e30, -np.inf, -200.0], dtype=np.float32))
    assert np.all((low > 0) & (low < 1e-37))
    assert _ex2_poly(np.array([0.0], dtype=np.float32))[0] == 1.0
