"""The quantizers divide the NVFP4 block amax by 6 with one product by RN(1/6)
and one fused correction (the division-by-a-known-divisor method of
Brisebarre, Muller and Raina, IEEE Trans. Computers 53(8), 2004) for finite
x >= 2^-125, and with the division itself elsewhere. This checks, for every
fp32 in that range, that the two steps give the correctly rounded quotient
(IEEE single precision on the host: the same products, fused multiply-adds
and divisions the kernel's __fmul_rn / __fmaf_rn / __fdiv_rn perform)."""
import os
import subprocess
import shutil

import pytest

import helpers

SRC = r"""
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>
int main(void) {
    const float C = 1.0f / 6.0f;
    const uint32_t lo = 0x01000000u;   /* 2^-125 */
    const uint32_t hi = 0x7F800000u;   /* +inf, excluded */
    unsigned long long bad = 0;
    #pragma omp parallel for reduction(+:bad) schedule(static)
    for (long long i = lo; i < (long long)hi; ++i) {
        float x, q, r, y, ref;
        uint32_t u = (uint32_t)i, a, b;
        memcpy(&x, &u, 4);
        q = x * C;
        r = fmaf(-q, 6.0f, x);
        y = fmaf(r, C, q);
        ref = x / 6.0f;
        memcpy(&a, &y, 4);
        memcpy(&b, &ref, 4);
        bad += (a != b);
    }
    printf("%llu\n", bad);
    return 0;
}
"""


def test_divide_by_six_is_correctly_rounded_above_2_pow_minus_125():
    d = helpers.scratch_dir("div6_")
    try:
        c, exe = os.path.join(d, "div6.c"), os.path.join(d, "div6")
        with open(c, "w") as f:
            f.write(SRC)
        flags = ["-O2", "-fopenmp", "-ffp-contract=off", "-march=native"]
        try:
            subprocess.check_call(["gcc", *flags, c, "-o", exe, "-lm"])
        except (OSError, subprocess.CalledProcessError):
            pytest.skip("no host C compiler with OpenMP")
        out = subprocess.check_output([exe], text=True, timeout=600)
    finally:
        shutil.rmtree(d, ignore_errors=True)
    assert int(out.strip()) == 0
