"""The quantizers divide the NVFP4 block amax (x >= 0) by 6 without a
division: for finite x >= 2^-125 with one product by RN(1/6) and one fused
correction (the division-by-a-known-divisor method of Brisebarre, Muller and
Raina, IEEE Trans. Computers 53(8), 2004); below 2^-125, where the quotient is
subnormal, as round-half-even(N / 6) * 2^-149 with N the bits of x (x =
N * 2^-149 for exponent fields 0 and 1). This checks, for every non-negative
fp32 below +inf, that the result is the correctly rounded quotient (IEEE
single precision on the host: the same products and fused multiply-adds the
kernel's __fmul_rn / __fmaf_rn perform, against the host's division)."""
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
    unsigned long long bad = 0, bad_sub = 0;
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
    #pragma omp parallel for reduction(+:bad_sub) schedule(static)
    for (long long i = 0; i < (long long)lo; ++i) {
        uint32_t n = (uint32_t)i, qi = n / 6u, rem = n - 6u * qi, b;
        uint32_t y = qi + ((2u * rem > 6u || (2u * rem == 6u && (qi & 1u) != 0u)) ? 1u : 0u);
        float x, ref;
        memcpy(&x, &n, 4);
        ref = x / 6.0f;
        memcpy(&b, &ref, 4);
        bad_sub += (y != b);
    }
    printf("%llu %llu\n", bad, bad_sub);
    return 0;
}
"""


def test_divide_by_six_is_correctly_rounded():
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
    assert [int(v) for v in out.split()] == [0, 0]
