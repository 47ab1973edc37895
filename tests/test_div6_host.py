"""The quantizer's block-scale division by 6, checked exhaustively on the host (CPU only).

The kernels form RN(amax_b / 6) (reading R4's op order) without a division routine:
with y = RN(1/6), q = RN(amax_b * y), r = fma(-q, 6, amax_b) (exact), RN(q + r * y) by
one more FMA -- the correction step for division by a known constant (Markstein;
Brisebarre, Muller and Raina, IEEE TC 2004).  The kernels use it for amax_b >= 2^-125
and IEEE division below.  This test repeats the three operations in C (binary32, round
to nearest even, fused multiply-add from the C library) for every finite fp32 value
>= 2^-125 and compares them bit for bit with IEEE division, and confirms that smaller
values do need the division."""
import os
import subprocess
import tempfile

SRC = r"""
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>
static float f_of(uint32_t b) { float f; memcpy(&f, &b, 4); return f; }
static float via_fma(float a) {
    const float y = 1.0f / 6.0f;
    const float q = a * y;
    return fmaf(fmaf(-q, 6.0f, a), y, q);
}
int main(void) {
    const uint32_t lo = 0x01000000u;  /* 2^-125 */
    long long bad_hi = 0, bad_lo = 0;
    #pragma omp parallel for reduction(+ : bad_hi) schedule(static)
    for (int64_t u = lo; u < 0x7F800000ll; ++u) {
        const float a = f_of((uint32_t)u), r = via_fma(a), ref = a / 6.0f;
        if (memcmp(&r, &ref, 4) != 0) ++bad_hi;
    }
    for (uint32_t u = 0; u < lo; ++u) {
        const float a = f_of(u), r = via_fma(a), ref = a / 6.0f;
        if (memcmp(&r, &ref, 4) != 0) ++bad_lo;
    }
    printf("%lld %lld\n", bad_hi, bad_lo);
    return 0;
}
"""


def test_fma_division_by_6_is_exact_above_2_pow_minus_125():
    with tempfile.TemporaryDirectory() as d:
        c, exe = os.path.join(d, "div6.c"), os.path.join(d, "div6")
        with open(c, "w") as f:
            f.write(SRC)
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
                               c, "-o", exe, "-lm"])
        bad_hi, bad_lo = map(int, subprocess.check_output([exe], timeout=600).split())
    assert bad_hi == 0          # every a >= 2^-125: bit-identical to IEEE a / 6
    assert bad_lo > 0           # below it the correction is not enough: the kernels divide
