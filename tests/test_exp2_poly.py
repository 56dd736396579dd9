"""The FMA-pipe exponential the prefill softmax uses for a share of its scores (exp2_poly2 in
csrc/common.cuh): its constants are read from the source and the same float32 steps are replayed
on the CPU -- round-to-nearest through x + 1.5 * 2^23, the cubic in f = x - round(x), and the
integer add of round(x) << 23 to the exponent field -- against 2^x in double precision."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(__file__)), "position_agnostic_paged_b200", "csrc",
                   "common.cuh")


def _coeffs():
    txt = open(SRC).read()
    m = re.search(r"kExp2C0 = ([0-9.e+-]+)f, kExp2C1 = ([0-9.e+-]+)f, kExp2C2 = ([0-9.e+-]+)f, "
                  r"kExp2C3 = ([0-9.e+-]+)f", txt)
    assert m, "coefficients not found"
    return [np.float32(float(v)) for v in m.groups()]


def _exp2_poly(x):
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-120.0))
    r = np.float32(12582912.0)
    t = (x + r).astype(np.float32)
    n = (t - r).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = (f * c3 + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = (t.view(np.uint32).astype(np.uint64) * 8388608 + p.view(np.uint32).astype(np.uint64)) % (1 << 32)
    return bits.astype(np.uint32).view(np.float32), x


def test_relative_error_over_the_softmax_range():
    x = np.linspace(-120.0, 64.0, 1_000_001, dtype=np.float32)
    y, xc = _exp2_poly(x)
    rel = np.abs(y.astype(np.float64) / np.exp2(xc.astype(np.float64)) - 1.0)
    assert rel.max() <= 7.6e-5          # the cubic's minimax error on [-1/2, 1/2]; bf16 rounding is 2^-9
    # exact at integers up to the cubic's constant term
    yi, _ = _exp2_poly(np.arange(-8, 9, dtype=np.float32))
    np.testing.assert_allclose(yi, np.exp2(np.arange(-8.0, 9.0)), rtol=7.6e-5)


def test_masked_scores_give_tiny_positive_values_that_the_kernel_discards():
    """-inf (a masked score) is raised to -120: 2^-120, far below any visible weight (>= 2^-8 next
    to the row maximum); rows that see no key at all are zeroed by their -inf running maximum."""
    y, _ = _exp2_poly(np.array([-np.inf, -1e30, -500.0], np.float32))
    assert np.all(y == np.float32(2.0 ** -120 * 0.99992807)) or np.allclose(y, 2.0 ** -120, rtol=1e-4)
    assert np.all(y > 0) and np.all(y < 2.0 ** -119)
