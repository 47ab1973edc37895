"""The stochastic-rounding arithmetic of the quantize kernels, emulated exactly on
the host and compared with the oracle's rounding rule (CPU only).

The kernels do not select grid neighbours per element.  They clamp a = min(|v|, 6)
and map it through the concave code-space map c(a) = min(2a, a + 2, a/2 + 4), which
is affine between grid points and sends the E2M1 grid {0, .5, 1, 1.5, 2, 3, 4, 6} to
the codes 0..7 (c(6) = 7, so no further cap is needed).  So floor(c) is the code of the lower neighbour and frac(c) is
the round-up probability p, and the code is floor(c) + [r < p * 2^16] =
(ceil(c * 2^16) + 65535 - r) >> 16 for the 16-bit draw r.  Each branch of the
minimum is one fp32 FMA rounded upward, with addend 2^23 + offset * 2^16 + 65535.
The sums are integers below 2^24, so the only rounding is the ceiling, and the
minimum commutes with it (the kernels evaluate two elements per packed fp32x2 FMA
and take the minimum of the three branches in one three-input min).  The float's
bits minus r then hold the code in bits 16-18.

This test repeats those steps with exact rational arithmetic for the upward
rounding and compares the code with the oracle's rule ("round up iff r < p * 2^16",
sign bit copied).  It covers:
- every grid point and its float neighbours;
- random values;
- tiny and saturating values;
- draws at both ends and in the middle.
"""
import math
from fractions import Fraction

import numpy as np

from oracle import oracle as ora

SLOPES = (131072.0, 65536.0, 32768.0)  # 2^16 * (2, 1, 1/2)
ADDENDS = (8388608 + 65535, 8388608 + 2 * 65536 + 65535, 8388608 + 4 * 65536 + 65535)


def fma_round_up(a, b, c):
    """fp32 a*b + c rounded toward +inf (exact rational evaluation)."""
    exact = Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c))
    if exact > Fraction(float(np.finfo(np.float32).max)):
        return np.float32(np.inf)  # rounding up past the largest float gives +inf
    x = np.float32(float(exact))
    while Fraction(float(x)) < exact:
        x = np.nextafter(x, np.float32(np.inf))
    while Fraction(float(np.nextafter(x, np.float32(-np.inf)))) >= exact:
        x = np.nextafter(x, np.float32(-np.inf))
    return x


def kernel_code(v, r):
    v = np.float32(v)
    a = np.float32(min(abs(float(v)), 6.0))
    t = min(fma_round_up(a, s, c) for s, c in zip(SLOPES, ADDENDS))
    bits = int(np.float32(t).view(np.uint32))
    assert bits >> 23 == 0x96  # the value lies in [2^23, 2^24): the code is in bits 16-18
    code = ((bits - r) >> 16) & 7
    return code | (8 if np.signbit(v) else 0)


def test_code_map_equals_round_up_rule():
    rng = np.random.default_rng(7)
    vals = list(rng.uniform(-7, 7, 300).astype(np.float32))
    vals += list((rng.standard_normal(60) * 1e-3).astype(np.float32))
    for g in (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0):
        for sgn in (1.0, -1.0):
            x = np.float32(sgn * g)
            vals += [x, np.nextafter(x, np.float32(10)), np.nextafter(x, np.float32(-10))]
    vals += [np.float32(-0.0), np.float32(1e-45), np.float32(-1e-45), np.float32(6.5),
             np.float32(-1e30), np.float32(3e38)]
    draws = list(range(0, 65536, 2053)) + [0, 1, 2, 32767, 32768, 65534, 65535]
    bad = [(float(v), r) for v in vals for r in draws if kernel_code(v, r) != ora.e2m1_encode_sr(v, r)]
    assert not bad, bad[:5]


def test_code_map_probability_is_exact():
    """Between each pair of grid neighbours, the draws r < ceil(p * 2^16) round up and
    the others round down, so the round-up share is p at the resolution of a 16-bit
    draw.  The code cannot increase with r, so the two draws at the boundary and the
    two extremes fix the whole partition."""
    grid = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)
    for lo, hi in zip(grid, grid[1:]):
        for frac in (0.3, 0.5, 0.77):
            v = np.float32(lo + frac * (hi - lo))
            p = (Fraction(float(v)) - Fraction(lo)) / (Fraction(hi) - Fraction(lo))
            b = math.ceil(p * 65536)
            up, down = grid.index(hi), grid.index(lo)
            assert kernel_code(v, 0) == up and kernel_code(v, b - 1) == up, (v, b)
            assert kernel_code(v, b) == down and kernel_code(v, 65535) == down, (v, b)
