"""Pins of the CPU oracle against facts fixed outside it.

Each ``check_*`` raises AssertionError when the oracle disagrees with what the
pages, the mathematics or an independent library routine fix. The checks are
plain functions so that ``test_oracle_pins`` runs them on the oracle and
``test_oracle_mutations`` runs them on copies of the oracle with a planted
mistake (each mutant must fail at least one check).

Sources cited: the pages "Quartet II - obuchenie v NVFP4 s tochnymi
nesmeshchyonnymi gradientami", "New AMD paper overturns conventional wisdom:
FP4 training..." (sections "Chto takoe MXFP4", "Poiskovaya eksperimental'naya
rabota") and "NVIDIA sozdala metod obucheniya neyrosetey v 4-bit tochnosti"
(section "Kak eto rabotaet").
"""
from __future__ import annotations

import json
import os
import subprocess
from fractions import Fraction

import numpy as np
import torch

import helpers
import oracle as O
from fp4_precision_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# number formats

def check_e2m1_value_set():
    """The E2M1 magnitude set is {0, 0.5, 1, 1.5, 2, 3, 4, 6} with a sign bit."""
    g = golden("formats.json")
    vals = sorted({O.e2m1_value(c) for c in range(16)})
    expect = sorted({s * m for m in g["e2m1_magnitudes"] for s in (1.0, -1.0)})
    assert vals == expect, (vals, expect)
    for c in range(8):
        assert O.e2m1_value(c) == g["e2m1_magnitudes"][c]
        assert O.e2m1_value(c | 8) == -g["e2m1_magnitudes"][c]


def _rne_e2m1_reference(u: float) -> float:
    """Independent formulation: E2M1 is a binary float with one mantissa bit,
    emin 0 (subnormal step 0.5) and largest finite 6. Python's round() is
    round-half-to-even, applied to the value in units of the local step."""
    a = abs(u)
    if a < 2.0:
        m = round(a * 2) / 2
    elif a < 4.0:
        m = float(round(a))
    else:
        m = 2.0 * round(a / 2)
    m = min(m, 6.0)
    return -m if (u < 0 and m != 0) else m


def check_e2m1_rtn_exhaustive_bf16():
    """RTN on every bf16 value in [-8, 8] equals the independent RNE formulation,
    and every tie listed in the golden file goes to the even code."""
    bits = np.arange(0, 1 << 16, dtype=np.uint32)
    vals = (bits << 16).astype(np.uint32).view(np.float32)
    vals = vals[np.isfinite(vals) & (np.abs(vals) <= 8.0)]
    for u in vals.tolist():
        got = O.e2m1_value(O.e2m1_rtn(u))
        ref = _rne_e2m1_reference(u)
        assert got == ref, (u, got, ref)
        if got == 0.0:
            assert O.e2m1_rtn(u) == 0, ("-0 must encode as code 0", u)
    for u, expect in golden("formats.json")["e2m1_rtn_ties"]:
        assert O.e2m1_value(O.e2m1_rtn(u)) == expect, (u, expect)
        assert O.e2m1_value(O.e2m1_rtn(-u)) == -expect
    for u in (6.5, 7.0, 100.0, 3.0e38):
        assert O.e2m1_rtn(u) == 7 and O.e2m1_rtn(-u) == 15


def check_e4m3_matches_torch():
    """Decoding all 256 E4M3 codes and RN-encoding fp32 values in [0, 448]
    (every grid value, every midpoint and its neighbours, random values) agree
    with torch's float8_e4m3fn conversion; values at or above 448 saturate."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([O.e4m3_value(c) for c in range(256)])
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])
    grid = np.array([O.e4m3_value(c) for c in range(0x7F)], dtype=np.float64)
    mids = (grid[:-1] + grid[1:]) / 2
    probe = np.concatenate([grid, mids, np.nextafter(mids.astype(np.float32), np.float32(0)),
                            np.nextafter(mids.astype(np.float32), np.float32(1000)),
                            np.exp(np.random.default_rng(0).uniform(np.log(1e-12), np.log(448), 4000))])
    probe = probe.astype(np.float32)
    probe = probe[(probe >= 0) & (probe <= 448)]
    tref = torch.from_numpy(probe).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    tgot = np.array([O.e4m3_rne_sat(float(t)) for t in probe], dtype=np.uint8)
    assert np.array_equal(tref, tgot), probe[tref != tgot][:10]
    for t in (448.0, 449.0, 464.0, 1e6, 3e38):
        assert O.e4m3_rne_sat(t) == 0x7E


def check_e8m0_matches_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    got = np.array([O.e8m0_value(c) for c in range(256)])
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])


# ---------------------------------------------------------------------------
# Philox

_PHILOX_HARNESS = r"""
#include <ATen/core/PhiloxRNGEngine.h>
#include <cstdio>
int main() {
  unsigned long long seed, sub, off;
  while (std::scanf("%llu %llu %llu", &seed, &sub, &off) == 3) {
    at::Philox4_32 e(seed, sub, off);
    unsigned a = e(), b = e(), c = e(), d = e();
    std::printf("%u %u %u %u\n", a, b, c, d);
  }
}
"""
_philox_ref_bin = None


def _torch_philox(cases):
    """Philox4x32-10 from torch's header-only engine (key = seed, counter =
    (offset lo, offset hi, subsequence lo, subsequence hi))."""
    global _philox_ref_bin
    if _philox_ref_bin is None:
        d = helpers.scratch_dir("philox_ref_")
        src = os.path.join(d, "ref.cpp")
        with open(src, "w") as f:
            f.write(_PHILOX_HARNESS)
        inc = os.path.join(os.path.dirname(torch.__file__), "include")
        out = os.path.join(d, "ref")
        subprocess.check_call(["g++", "-std=c++17", "-O1", "-I", inc, src, "-o", out])
        _philox_ref_bin = out
    text = "".join(f"{s} {sub} {off}\n" for s, sub, off in cases)
    res = subprocess.run([_philox_ref_bin], input=text, capture_output=True, text=True, check=True)
    return [tuple(int(v) for v in line.split()) for line in res.stdout.strip().splitlines()]


def check_philox_matches_torch_engine():
    rng = np.random.default_rng(1)
    cases, ours = [], []
    for _ in range(200):
        c = [int(v) for v in rng.integers(0, 2**32, 4, dtype=np.uint64)]
        k = [int(v) for v in rng.integers(0, 2**32, 2, dtype=np.uint64)]
        cases.append((k[0] | (k[1] << 32), c[2] | (c[3] << 32), c[0] | (c[1] << 32)))
        ours.append(tuple(int(v) for v in O.philox4x32_10(c, k)))
    cases.append((0, 0, 0))
    ours.append(tuple(int(v) for v in O.philox4x32_10([0, 0, 0, 0], [0, 0])))
    assert _torch_philox(cases) == ours
    # the stream layout: word i%4 of counter (i/4, tag | stream<<4, 0)
    seed, tag, stream = 0x1234_5678_9ABC_DEF0, O.TAG_SCALE, 5
    ref = _torch_philox([(seed, tag | (stream << 4), i // 4) for i in range(0, 64, 4)])
    for i in range(64):
        assert O.random_word(seed, tag, stream, i) == ref[i // 4][i % 4]


def check_element_uniform_layout():
    """Element SR uniforms (16 bits each): element i takes half (i mod 2), low
    half first, of word floor(i/2) of its stream, i.e. of word (i/2) mod 4 of
    the Philox block with counter (i/8, TAG_ELEMENT | stream << 4, 0), scaled
    by 2^-16 — checked against torch's Philox engine for 128 elements."""
    seed, stream = 0x0F1E_2D3C_4B5A_6978, 9
    ref = _torch_philox([(seed, O.TAG_ELEMENT | (stream << 4), i // 8) for i in range(0, 128, 8)])
    for i in range(128):
        w = ref[i // 8][(i // 2) % 4]
        half = (w >> (16 * (i % 2))) & 0xFFFF
        assert O.element_uniform(seed, stream, i) == half * 2.0**-16, i


# ---------------------------------------------------------------------------
# Hadamard

def check_sylvester_matches_scipy():
    import scipy.linalg
    for n in (2, 4, 8, 16, 32):
        H = O.hadamard_matrix(n).astype(np.int64)
        assert np.array_equal(H, scipy.linalg.hadamard(n)), n
        assert np.array_equal(H @ H.T, n * np.eye(n, dtype=np.int64)), n


def check_fwht_is_matrix_product():
    """FWHT(w) == H w exactly on small integers (sums exact in fp32) and to fp32
    rounding on Gaussian data; H H w = n w."""
    rng = np.random.default_rng(2)
    for n in (16, 32):
        H = O.hadamard_matrix(n).astype(np.float64)
        for _ in range(50):
            w = rng.integers(-1000, 1000, n).astype(np.float32)
            assert np.array_equal(O.fwht(w).astype(np.float64), H @ w.astype(np.float64))
            w = rng.standard_normal(n).astype(np.float32)
            assert np.allclose(O.fwht(w), H @ w, rtol=0, atol=1e-5 * np.abs(w).sum())
            assert np.allclose(O.fwht(O.fwht(w)), n * w, rtol=1e-5, atol=1e-5)


def check_rotation_orthonormal():
    """The rotation preserves the norm of every chunk, and the fp64 inverse
    (D H / sqrt(n)) recovers the input, for deterministic and random signs."""
    x = inputs.normal((8, 64), 1.0, 3, "rot")
    xf = x.float().numpy().astype(np.float64)
    for had in (O.HAD_DET16, O.HAD_DET32, O.HAD_RAND16, O.HAD_RAND32):
        n = O.HAD_N[had]
        v = O.rotate(x, had, O.ROW, 77, 3).astype(np.float64)
        nv = np.linalg.norm(v.reshape(8, -1, n), axis=2)
        nx = np.linalg.norm(xf.reshape(8, -1, n), axis=2)
        assert np.allclose(nv, nx, rtol=1e-6), had
        back = O.unrotate(v, had, 77, 3)
        assert np.allclose(back, xf, rtol=0, atol=1e-6), had
    # a random sign vector actually flips signs and depends on the seed
    assert O.sign_bits(1) != O.sign_bits(2)
    v_det = O.rotate(x, O.HAD_DET16, O.ROW)
    v_rnd = O.rotate(x, O.HAD_RAND16, O.ROW, 1)
    assert not np.array_equal(v_det, v_rnd)


# ---------------------------------------------------------------------------
# stochastic rounding

def check_sr_threshold_exact():
    """For values u with exact round-up probability p (a fraction with a power
    of two denominator), SR rounds up for exactly ceil(p * 2^24) of the 2^24
    uniforms rho = m 2^-24: it rounds up at m = n-1 and down at m = n."""
    rng = np.random.default_rng(4)
    probe = [0.1, 0.3, 0.74, 1.1, 1.9, 2.2, 3.3, 3.99, 4.5, 5.9, 5.99999]
    probe += rng.uniform(0, 6, 40).tolist()
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for u in probe:
        u = float(np.float32(u))
        a = Fraction(u)
        lo = max(g for g in grid if g <= a)
        hi = min(g for g in grid if g > a)
        p = (a - Fraction(lo)) / (Fraction(hi) - Fraction(lo))
        n = -((-p * 2**24).numerator // (p * 2**24).denominator)  # ceil
        for sgn in (1.0, -1.0):
            up = O.e2m1_value(O.e2m1_sr(sgn * u, 0.0 if n == 0 else (n - 1) * 2.0**-24))
            down = O.e2m1_value(O.e2m1_sr(sgn * u, n * 2.0**-24)) if n < 2**24 else None
            if n > 0:
                assert up == sgn * hi, (u, n, up)
            if down is not None:
                assert down == (sgn * lo if lo != 0 else 0.0), (u, n, down)
    for u in (6.0, 7.5, 1e9):
        assert O.e2m1_value(O.e2m1_sr(u, 0.999)) == 6.0


def check_sr_threshold_exact_16bit():
    """With the 16-bit element uniforms rho = m 2^-16, SR rounds up for exactly
    ceil(p * 2^16) of the 2^16 values: up at m = n - 1, down at m = n (p the
    exact fraction between the grid neighbours)."""
    rng = np.random.default_rng(14)
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    probe = [0.1, 0.3, 0.74, 1.1, 1.9, 2.2, 3.3, 3.99, 4.5, 5.9, 5.99999, 0.25 + 2.0**-20, 1.0 + 2.0**-17]
    for u in probe + rng.uniform(0, 6, 40).tolist():
        u = float(np.float32(u))
        a = Fraction(u)
        lo = max(g for g in grid if g <= a)
        hi = min(g for g in grid if g > a)
        p = (a - Fraction(lo)) / (Fraction(hi) - Fraction(lo))
        n = -((-p * 2**16).numerator // (p * 2**16).denominator)  # ceil
        if n > 0:
            assert O.e2m1_value(O.e2m1_sr(u, (n - 1) * 2.0**-16)) == hi, (u, n)
        if n < 2**16:
            assert O.e2m1_value(O.e2m1_sr(u, n * 2.0**-16)) == lo, (u, n)


def check_e4m3_sr_threshold_exact():
    rng = np.random.default_rng(5)
    grid = [Fraction(O.e4m3_value(c)) for c in range(0x7F)]
    for t in rng.uniform(0, 440, 60).tolist() + [1e-4, 0.0019, 0.3, 447.0]:
        t = float(np.float32(t))
        a = Fraction(t)
        i = max(j for j, g in enumerate(grid) if g <= a)
        p = (a - grid[i]) / (grid[i + 1] - grid[i])
        n = -((-p * 2**24).numerator // (p * 2**24).denominator)
        if n > 0:
            assert O.e4m3_sr(t, (n - 1) * 2.0**-24) == i + 1, t
        if n < 2**24:
            assert O.e4m3_sr(t, n * 2.0**-24) == i, t


def check_e8m0_sr_threshold_exact():
    """Stochastic rounding onto powers of two (the Quartet II scale step of
    MXFP4): for t in [2^e, 2^(e+1)) the round-up probability is p = (t - 2^e) /
    2^e, exact as a Fraction; the code is e + 127, plus one for exactly the
    ceil(p 2^24) uniforms below p. Exponents are clamped to [-127, 127], and a
    power of two never rounds up."""
    rng = np.random.default_rng(6)
    ts = [float(np.float32(v)) for v in rng.uniform(0.5, 2.0, 20) * np.exp2(rng.integers(-130, 120, 20))]
    ts += [1.0, 1.5, 3.0, 1.9999999, 0.75, 2.0**-127 * 1.25, 2.0**127 * 1.5, 2.0**-130 * 1.7]
    for t in ts:
        t = float(np.float32(t))
        a = Fraction(t)
        e = a.numerator.bit_length() - a.denominator.bit_length()
        if Fraction(2) ** e > a:
            e -= 1
        lo = Fraction(2) ** e
        p = (a - lo) / lo
        n = -((-p * 2**24).numerator // (p * 2**24).denominator)  # ceil
        clamp = lambda k: min(max(k, -127), 127) + 127  # noqa: E731
        if n > 0:
            assert O.e8m0_sr(t, (n - 1) * 2.0**-24) == clamp(e + 1), (t, n)
        if n < 2**24:
            assert O.e8m0_sr(t, n * 2.0**-24) == clamp(e), (t, n)
    for e in (-20, 0, 5, 100):
        assert O.e8m0_sr(2.0**e, 0.0) == e + 127
        assert O.e8m0_sr(2.0**e, 1.0 - 2.0**-24) == e + 127


def _stats_over_seeds(x, fmt, rnd, had, n_seeds, rot_varies):
    """Mean and variance of the de-rotated estimate over seeds, and the mean
    product of the errors of neighbouring elements (j, j+1)."""
    acc = None
    xf = x.float().numpy().astype(np.float64)
    for s in range(n_seeds):
        rot = 1000 + s if rot_varies else 7
        q = O.quantize(x, fmt, rnd, had, O.ROW, rot, 0, s, 0)
        est = O.unrotate(O.dequantize(q), had, rot, 0)
        if acc is None:
            acc, acc2, accx = np.zeros_like(est), np.zeros_like(est), np.zeros_like(est[:, :-1])
        acc += est
        acc2 += est * est
        err = est - xf
        accx += err[:, :-1] * err[:, 1:]
    mean = acc / n_seeds
    var = np.maximum(acc2 / n_seeds - mean * mean, 0.0)
    return mean, var, accx / n_seeds


def check_sr_unbiased_rtn_biased():
    """[Quartet II], [AMD MXFP4] "Poiskovaya...": stochastic rounding makes the
    estimate unbiased. Over 10^4 seeds the mean error of every non-clipped
    element is within 4 standard errors of 0; RTN, deterministic, fails the
    same test on most elements. The rounding noise of neighbouring elements
    is uncorrelated (every element draws its own uniform)."""
    x = inputs.normal((8, 64), 1.0, 5, "sr")
    xf = x.float().numpy().astype(np.float64)
    for fmt in (O.NVFP4, O.MXFP4):
        n = 10_000
        mean, var, cross = _stats_over_seeds(x, fmt, O.SR, O.HAD_NONE, n, False)
        q = O.quantize(x, fmt, O.RTN, O.HAD_NONE, O.ROW)
        step = np.repeat(O.scale_values(q), O.BLOCK[fmt], axis=1) * (q.g if fmt == O.NVFP4 else 1.0)
        clipped = np.abs(xf) > 6.0 * step * (1 - 2.0**-20)
        se = np.sqrt(var / n + (2.0**-20 * np.abs(xf)) ** 2) + 1e-300
        z = np.abs(mean - xf) / se
        frac = np.mean(z[~clipped] < 4.0)
        assert frac >= 0.99, (fmt, frac)
        # the rounding noise of neighbouring elements is uncorrelated
        b = mean - xf
        cov = cross - b[:, :-1] * b[:, 1:]
        sd = np.sqrt(var[:, :-1] * var[:, 1:])
        both = (sd > 0) & ~clipped[:, :-1] & ~clipped[:, 1:]
        corr = cov[both] / sd[both]
        assert abs(np.mean(corr)) < 0.02 and np.mean(np.abs(corr) < 0.05) > 0.95, (fmt, np.mean(corr))
        rtn = O.dequantize(q)
        z_rtn = np.abs(rtn - xf) / (2.0**-20 * np.abs(xf) + 1e-300)
        assert np.mean(z_rtn[~clipped] < 4.0) < 0.5


def check_quartet2_projection_unbiased():
    """[Quartet II]: with the renormalisation stochastically rounded into the
    scale, the quantized block is unbiased along the block itself: the mean
    over rounding seeds of <x_hat_b, v_b> / <v_b, v_b> is 1 for every block
    (v the rotated block). RTN codes with the plain RTN scale are not."""
    x = inputs.normal((8, 128), 1.0, 6, "q2")
    for fmt, had in ((O.NVFP4, O.HAD_RAND16), (O.MXFP4, O.HAD_RAND32), (O.NVFP4, O.HAD_NONE)):
        nb = O.BLOCK[fmt]
        v = O.rotate(x, had, O.ROW, 7, 0).astype(np.float64)
        vb = v.reshape(8, -1, nb)
        vv = np.sum(vb * vb, axis=2)
        n = 4000
        acc = np.zeros_like(vv)
        acc2 = np.zeros_like(vv)
        for s in range(n):
            q = O.quantize(x, fmt, O.QUARTET2, had, O.ROW, 7, 0, s, 0)
            proj = np.sum(O.dequantize(q).reshape(8, -1, nb) * vb, axis=2) / vv
            acc += proj
            acc2 += proj * proj
        mean = acc / n
        # floor: one scale step (at most 2^-3 relative for E4M3, 1 for E8M0) in n draws
        floor = (2.0**-3 if fmt == O.NVFP4 else 1.0) / n
        se = np.sqrt(np.maximum(acc2 / n - mean * mean, 0) / n) + floor
        # blocks whose renormalised scale S * alpha reaches 448 saturate (biased by design)
        q2 = O.quantize(x, fmt, O.QUARTET2, had, O.ROW, 7, 0, 0, 0)
        q_rtn = O.quantize(x, fmt, O.RTN, had, O.ROW, 7, 0)
        unclipped = O.scale_values(q_rtn) * q2.alpha < (448.0 if fmt == O.NVFP4 else 2.0**127)
        frac = np.mean((np.abs(mean - 1.0) / se < 4.0)[unclipped])
        assert frac >= 0.98, (fmt, had, frac)
        q = O.quantize(x, fmt, O.RTN, had, O.ROW, 7, 0)
        proj_rtn = np.sum(O.dequantize(q).reshape(8, -1, nb) * vb, axis=2) / vv
        assert np.mean(np.abs(proj_rtn - 1.0) / se < 4.0) < 0.5, fmt


def check_quartet2_error_half_of_sr():
    """[Quartet II]: rounding only the renormalised scales stochastically (the
    element codes stay RTN) leaves about half the total error of per-element
    stochastic rounding. On N(0,1) data with and without a random 16x16
    rotation the mean squared error of the NVFP4 reconstruction (rotated
    domain, 4 rounding seeds) is within 0.4-0.6 of SR's; the part added by the
    scale rounding (over RTN) is at least 20x smaller than SR's (measured about
    30x; the page says about two orders of magnitude)."""
    ratio = golden("pages.json")["quartet2_error_vs_plain_sr"]
    x = inputs.normal((256, 1024), 1.0, 9, "mse")
    for had in (O.HAD_RAND16, O.HAD_NONE):
        v = O.rotate(x, had, O.ROW, 5, 0).astype(np.float64)
        mse = {}
        for rnd in (O.RTN, O.SR, O.QUARTET2):
            mse[rnd] = np.mean([np.mean((O.dequantize(O.quantize(x, O.NVFP4, rnd, had, O.ROW, 5, 0, 100 + s, 0))
                                         - v) ** 2) for s in range(4)])
        assert abs(mse[O.QUARTET2] / mse[O.SR] - ratio) < 0.1, mse
        assert (mse[O.SR] - mse[O.RTN]) > 20 * (mse[O.QUARTET2] - mse[O.RTN]) > 0, mse


def check_quartet2_alpha_range():
    """[Quartet II]: the renormalisation is of order 0.94-1.06. On N(0,1) data
    with a random 16x16 rotation at least 90% of the NVFP4 blocks' alpha fall in
    that range and all lie within [0.8, 1.25]."""
    lo, hi = golden("pages.json")["quartet2_alpha_range"]
    x = inputs.normal((256, 256), 1.0, 7, "alpha")
    q = O.quantize(x, O.NVFP4, O.QUARTET2, O.HAD_RAND16, O.ROW, 3, 0, 4, 0)
    a = q.alpha.ravel()
    assert np.mean((a >= lo) & (a <= hi)) >= 0.90
    assert a.min() > 0.8 and a.max() < 1.25
    # the scale codes changed by SR stay within one E4M3 step of S * alpha
    q_rtn = O.quantize(x, O.NVFP4, O.RTN, O.HAD_RAND16, O.ROW, 3, 0)
    s_rtn = O.scale_values(q_rtn).ravel()
    s_q2 = O.scale_values(q).ravel()
    t = s_rtn * a
    assert np.all(s_q2 <= t * (1 + 2.0**-3) + 1e-30) and np.all(s_q2 >= t * (1 - 2.0**-3))


def check_quartet2_alpha_is_the_projection():
    """[Quartet II]: the renormalisation of a block is the projection
    <u, u> / <u, q> of its scaled values u on their RTN values q. Recomputed
    here in fp64 from the oracle's own RTN output (u = rotated block / (S g),
    q = the E2M1 values of its codes), the oracle's fp32 alpha agrees to within
    the rounding of its fp32 sums (all terms u_j q_j share a sign, so nothing
    cancels): 2^-18 relative. A term, index or operand wrong anywhere in the
    two sums moves alpha by far more. Also: Quartet II keeps the RTN codes."""
    x = inputs.normal((32, 256), 1.0, 21, "alpha_exact")
    for fmt, had in ((O.NVFP4, O.HAD_RAND16), (O.NVFP4, O.HAD_NONE), (O.MXFP4, O.HAD_RAND32), (O.MXFP4, O.HAD_DET32)):
        nb = O.BLOCK[fmt]
        q_rtn = O.quantize(x, fmt, O.RTN, had, O.ROW, 9, 0)
        q2 = O.quantize(x, fmt, O.QUARTET2, had, O.ROW, 9, 0, 13, 0)
        assert np.array_equal(q2.codes, q_rtn.codes)
        v = O.rotate(x, had, O.ROW, 9, 0).astype(np.float64)
        step = O.scale_values(q_rtn) * (np.float64(q_rtn.g) if fmt == O.NVFP4 else 1.0)
        u = v.reshape(32, -1, nb) / step[:, :, None]
        e2m1 = np.array([O.e2m1_value(c) for c in range(16)])
        q = e2m1[O.unpack_codes(q_rtn.codes)].reshape(32, -1, nb)
        num, den = np.sum(u * u, axis=2), np.sum(u * q, axis=2)
        ok = den > 0
        assert ok.mean() > 0.99
        alpha = num[ok] / den[ok]
        rel = np.abs(q2.alpha[ok] / alpha - 1.0)
        assert rel.max() < 2.0**-18, (fmt, had, rel.max())


# ---------------------------------------------------------------------------
# scales and reconstruction

def check_nvfp4_scales():
    """NVFP4: g * 2688 recovers the rotated tensor's amax; each block's max
    element lands near the top of the E2M1 grid (|amax_b / (S g)| within
    E4M3 rounding of 6); RTN error of non-clipped elements is at most half a
    grid gap times the block step S g ([AMD MXFP4] "Chto takoe MXFP4": x is
    reconstructed as scale times a round-to-nearest FP4 value)."""
    x = inputs.workload("sweep")["T"][:256, :512]
    for had in (O.HAD_NONE, O.HAD_DET16, O.HAD_RAND32):
        v = O.rotate(x, had, O.ROW, 9, 0).astype(np.float64)
        q = O.quantize(x, O.NVFP4, O.RTN, had, O.ROW, 9, 0)
        amax = np.abs(v).max()
        assert abs(q.g * 2688.0 - amax) <= amax * 2.0**-22
        S = O.scale_values(q)
        step = S * q.g
        amax_b = np.abs(v).reshape(256, -1, 16).max(axis=2)
        ok = step > 0
        ratio = amax_b[ok] / step[ok]
        assert np.all(ratio <= 6.0 * (1 + 2.0**-4) * (1 + 2.0**-20))
        assert np.all(ratio[amax_b[ok] > amax * 2.0**-6] >= 6.0 * (1 - 2.0**-4) * (1 - 2.0**-20))
        xhat = O.dequantize(q)
        stepe = np.repeat(step, 16, axis=1)
        u = np.abs(v) / np.where(stepe > 0, stepe, 1)
        gap = np.where(u < 2, 0.5, np.where(u < 4, 1.0, 2.0))
        nc = (u <= 6.0) & (stepe > 0)
        assert np.all(np.abs(v - xhat)[nc] <= (gap / 2 * stepe)[nc] * (1 + 2.0**-18))


def check_mxfp4_scales():
    """MXFP4 ([AMD MXFP4] "Chto takoe MXFP4": 32-element blocks share the
    largest exponent, E8M0): the block max scaled by 2^-E lies in [4, 8), i.e.
    E = floor(log2 amax_b) - 2 puts the block max in the top binade of E2M1."""
    x = inputs.workload("sweep")["T"][:128, :512]
    q = O.quantize(x, O.MXFP4, O.RTN, O.HAD_NONE, O.ROW)
    assert golden("pages.json")["mx_block_elements"] == O.BLOCK[O.MXFP4]
    v = x.float().numpy().astype(np.float64)
    amax_b = np.abs(v).reshape(128, -1, 32).max(axis=2)
    S = O.scale_values(q)
    nz = amax_b > 0
    r = amax_b[nz] / S[nz]
    assert np.all((r >= 4.0) & (r < 8.0))
    xhat = O.dequantize(q)
    err = np.abs(xhat - v)
    Se = np.repeat(S, 32, axis=1)
    u = np.abs(v) / Se
    gap = np.where(u < 2, 0.5, np.where(u < 4, 1.0, 2.0))
    nc = u <= 6.0
    assert np.all(err[nc] <= (gap / 2 * Se)[nc])
    assert np.all(np.abs(xhat[~nc]) == 6.0 * Se[~nc])


def check_mxfp4_round_up():
    """MXFP4 with the round-up shared exponent (a variant the pages leave open:
    [AMD MXFP4] "Chto takoe MXFP4" gives the shared exponent only as the
    block's largest one): E is the smallest exponent with amax_b <= 6 * 2^E, so
    the block max scaled by 2^-E lies in (3, 6] and no element clips. Where the
    floor rule already leaves the block max at or below 6 the two rules agree
    on the block's scale and codes; elsewhere the round-up exponent is one
    above the floor one. Worked blocks: max 7 (the floor rule clips it to 6)
    gets E = 1 and 7 / 2 = 3.5 rounds, ties to even, to code 6 (value 4, so 8
    after scaling), 1 / 2 = 0.5 to code 1; a block whose max is exactly 6 keeps
    E = 0 (and -0.75 rounds, ties to even, to code 2 with the sign bit)."""
    x = inputs.workload("sweep")["T"][:128, :512]
    qf = O.quantize(x, O.MXFP4, O.RTN, O.HAD_NONE, O.ROW)
    qr = O.quantize(x, O.MXFP4_RU, O.RTN, O.HAD_NONE, O.ROW)
    v = x.float().numpy().astype(np.float64)
    amax_b = np.abs(v).reshape(128, -1, 32).max(axis=2)
    nz = amax_b > 0
    ratio = amax_b[nz] / O.scale_values(qr)[nz]
    assert np.all((ratio > 3.0) & (ratio <= 6.0))
    fits = (amax_b <= 6.0 * O.scale_values(qf)) & nz
    assert fits.any() and (nz & ~fits).any()
    ef, er = qf.scales.astype(np.int64), qr.scales.astype(np.int64)
    assert np.all(er[fits] == ef[fits])
    assert np.all(er[nz & ~fits] == ef[nz & ~fits] + 1)
    cf = O.unpack_codes(qf.codes).reshape(128, -1, 32)
    cr = O.unpack_codes(qr.codes).reshape(128, -1, 32)
    assert np.array_equal(cf[fits], cr[fits])
    # no element clips: every reconstruction is within half a grid gap
    S = np.repeat(O.scale_values(qr), 32, axis=1)
    u = np.abs(v) / S
    gap = np.where(u < 2, 0.5, np.where(u < 4, 1.0, 2.0))
    assert np.all(u <= 6.0)
    assert np.all(np.abs(O.dequantize(qr) - v) <= gap / 2 * S)
    # worked blocks
    b = torch.zeros((1, 96), dtype=torch.float32)
    b[0, 0], b[0, 1], b[0, 32], b[0, 33] = 7.0, 1.0, 6.0, -0.75
    q = O.quantize(b.to(torch.bfloat16), O.MXFP4_RU, O.RTN, O.HAD_NONE, O.ROW)
    assert list(q.scales[0]) == [128, 127, 0]
    assert int(q.codes[0, 0]) == 0x16 and int(q.codes[0, 16]) == 0xA7 and not q.codes[0, 32:].any()


def check_zero_and_degenerate():
    """All-zero input: zero codes, zero NVFP4 scales, g = 1; E8M0 code 0."""
    z = torch.zeros((32, 64), dtype=torch.bfloat16)
    for fmt in (O.NVFP4, O.MXFP4):
        for rnd in (O.RTN, O.SR, O.QUARTET2):
            q = O.quantize(z, fmt, rnd, O.HAD_RAND16, O.ROW, 1, 0, 1, 0)
            assert not q.codes.any() and not q.scales.any() and q.g == 1.0
    e = O.quantize(torch.zeros((0, 64), dtype=torch.bfloat16), O.NVFP4, O.RTN, O.HAD_NONE, O.ROW)
    assert e.codes.shape == (0, 32) and e.g == 1.0


# ---------------------------------------------------------------------------
# orientation, determinism, GEMM

def check_col_is_row_of_transpose():
    x = inputs.normal((64, 96), 1.0, 8, "col")
    xt = x.t().contiguous()
    for fmt in (O.NVFP4, O.MXFP4):
        for rnd in (O.RTN, O.SR, O.QUARTET2):
            for had in (O.HAD_NONE, O.HAD_DET32, O.HAD_RAND16):
                a = O.quantize(x, fmt, rnd, had, O.COL, 5, 1, 6, 2)
                b = O.quantize(xt, fmt, rnd, had, O.ROW, 5, 1, 6, 2)
                assert np.array_equal(a.codes, b.codes) and np.array_equal(a.scales, b.scales)
                assert a.g == b.g


def check_seed_determinism():
    x = inputs.normal((16, 64), 1.0, 9, "det")
    a = O.quantize(x, O.NVFP4, O.SR, O.HAD_RAND16, O.ROW, 1, 0, 2, 0)
    b = O.quantize(x, O.NVFP4, O.SR, O.HAD_RAND16, O.ROW, 1, 0, 2, 0)
    c = O.quantize(x, O.NVFP4, O.SR, O.HAD_RAND16, O.ROW, 1, 0, 3, 0)
    d = O.quantize(x, O.NVFP4, O.SR, O.HAD_RAND16, O.ROW, 1, 0, 2, 1)
    assert np.array_equal(a.codes, b.codes)
    assert not np.array_equal(a.codes, c.codes) and not np.array_equal(a.codes, d.codes)


def check_gemm_brute_force():
    """Tiny GEMMs: the fp64 oracle equals the exact rational sum of products of
    the dequantized operands (exactly for MXFP4, to fp64 rounding of the
    tensor-scale factors for NVFP4)."""
    X = inputs.normal_with_outliers((8, 64), 10, "gx")
    W = inputs.normal_with_outliers((6, 64), 10, "gw")
    for fmt in (O.NVFP4, O.MXFP4):
        A = O.quantize(X, fmt, O.RTN, O.HAD_DET16, O.ROW)
        B = O.quantize(W, fmt, O.SR, O.HAD_DET16, O.ROW, 0, 0, 3, 0)
        D = O.gemm(A, B)
        abs_sum = np.abs(O.dequantize(A)) @ np.abs(O.dequantize(B)).T
        cA = O.unpack_codes(A.codes)
        cB = O.unpack_codes(B.codes)
        sA, sB = O.scale_values(A), O.scale_values(B)
        nb = O.BLOCK[fmt]
        for i in range(8):
            for j in range(6):
                acc = Fraction(0)
                for kk in range(64):
                    a = Fraction(O.e2m1_value(int(cA[i, kk]))) * Fraction(sA[i, kk // nb]) * Fraction(A.g)
                    b = Fraction(O.e2m1_value(int(cB[j, kk]))) * Fraction(sB[j, kk // nb]) * Fraction(B.g)
                    acc += a * b
                # MXFP4 products are powers of two times small integers: exact. An
                # NVFP4 product carries g_A g_B (2 x 24 bits): one fp64 rounding each.
                tol = 0 if fmt == O.MXFP4 else abs_sum[i, j] * Fraction(2) ** -50
                assert abs(Fraction(D[i, j]) - acc) <= tol, (fmt, i, j)


def check_hadamard_cancels_in_gemm():
    """Both operands rotated by the same H D along K: their product estimates
    X W^T. The rotated-quantized GEMM is within quantization noise of the fp64
    product of the bf16 inputs, and it is far from a product whose operands
    use different sign vectors."""
    X = inputs.normal((64, 256), 1.0, 11, "hx")
    W = inputs.normal((48, 256), 1.0, 11, "hw")
    ref = X.double().numpy() @ W.double().numpy().T
    A = O.quantize(X, O.NVFP4, O.RTN, O.HAD_RAND16, O.ROW, 5, 0)
    B = O.quantize(W, O.NVFP4, O.RTN, O.HAD_RAND16, O.ROW, 5, 0)
    err = np.linalg.norm(O.gemm(A, B) - ref) / np.linalg.norm(ref)
    assert err < 0.15, err
    B2 = O.quantize(W, O.NVFP4, O.RTN, O.HAD_RAND16, O.ROW, 5, 1)
    err2 = np.linalg.norm(O.gemm(A, B2) - ref) / np.linalg.norm(ref)
    assert err2 > 0.5, err2


ALL_CHECKS = [
    check_e2m1_value_set, check_e2m1_rtn_exhaustive_bf16, check_e4m3_matches_torch, check_e8m0_matches_torch,
    check_philox_matches_torch_engine, check_sylvester_matches_scipy, check_fwht_is_matrix_product,
    check_element_uniform_layout, check_rotation_orthonormal, check_sr_threshold_exact,
    check_sr_threshold_exact_16bit, check_e4m3_sr_threshold_exact,
    check_e8m0_sr_threshold_exact,
    check_sr_unbiased_rtn_biased, check_quartet2_projection_unbiased, check_quartet2_error_half_of_sr,
    check_quartet2_alpha_range, check_quartet2_alpha_is_the_projection,
    check_nvfp4_scales, check_mxfp4_scales, check_mxfp4_round_up, check_zero_and_degenerate, check_col_is_row_of_transpose,
    check_seed_determinism, check_gemm_brute_force, check_hadamard_cancels_in_gemm,
]
