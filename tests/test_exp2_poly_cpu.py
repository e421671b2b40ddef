"""The FMA-pipe exponential used in the SCA softmax (exp2_poly2 in
csrc/common.cuh), re-evaluated in float32 NumPy with the coefficients read
from the source, against the exact 2^x: relative error below 1e-4 on the
range the kernel uses (arguments <= 8 after the lazy max; large negative
arguments clamp to 2^-125; there is no upper clamp)."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "long_context_sequence_sca_b200", "csrc", "common.cuh")


def _coeffs():
    body = open(SRC).read().split("exp2_poly2(uint64_t x2)")[1].split("}\n")[0]
    vals = [float(v) for v in re.findall(r"pack2\(([0-9.e+-]+)f, \1f\)", body)]
    vals = [v for v in vals if abs(v) < 1.0]   # drop the rounding constants
    # order of appearance: c3, c2, c1, c0
    return np.float32(vals[0]), np.float32(vals[1]), np.float32(vals[2]), np.float32(vals[3])


def _poly_exp2(x):
    c3, c2, c1, c0 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-125))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = ((c3 * f + c2) * f + c1) * f + c0
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_poly_exp2_relative_error():
    x = np.linspace(-120, 8, 2_000_001, dtype=np.float32)
    got = _poly_exp2(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got / want - 1)) < 1e-4


def test_poly_exp2_clamps_large_negative_to_tiny():
    x = np.array([-np.inf, -1e30, -300.0, -126.0], dtype=np.float32)
    got = _poly_exp2(x)
    assert np.all(got > 0) and np.all(got < 1e-37)
