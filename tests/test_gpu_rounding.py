"""The quantizers' rounding steps, applied by the library's own device code
(qfp4_selftest_rounding) to chosen fp32 values, against the oracle's
definitions: E2M1 stochastic rounding and round-to-nearest ([NVIDIA NVFP4]
"Kak eto rabotaet"; [AMD MXFP4] "Chto takoe MXFP4"), E4M3 round-to-nearest and
stochastic rounding of the Quartet II scale, and the E8M0 variant ([Quartet
II]). The values sit on the grid points, on the stochastic-rounding thresholds
themselves (where the exact comparison decides) and on their neighbouring
floats, which random quantizer inputs reach only by chance; every code byte
must equal the oracle's."""
import numpy as np
import pytest
import torch

import oracle as O
from fp4_precision_b200 import qfp4 as Q

pytestmark = pytest.mark.gpu

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def neighbours(v: np.ndarray, k: int = 2) -> np.ndarray:
    """v with its k nearest floats on each side (positive values)."""
    out = [v]
    up, dn = v.copy(), v.copy()
    for _ in range(k):
        up = np.nextafter(up, np.float32(np.inf)).astype(np.float32)
        dn = np.nextafter(dn, np.float32(0)).astype(np.float32)
        out += [up, dn]
    return np.concatenate(out)


def run(op, x: np.ndarray, w: np.ndarray | None) -> np.ndarray:
    xd = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    wd = None if w is None else torch.from_numpy(np.ascontiguousarray(w, dtype=np.uint32).view(np.int32)).cuda()
    codes = Q.selftest_rounding(op, xd, wd)
    torch.cuda.synchronize()
    Q.status()
    return codes.cpu().numpy()


def check(got: np.ndarray, want: np.ndarray, x: np.ndarray, w):
    bad = np.flatnonzero(got != want)
    detail = [(float(x[i]), None if w is None else int(w[i]), int(got[i]), int(want[i])) for i in bad[:5]]
    assert bad.size == 0, f"{bad.size} of {got.size} codes differ (x, w, gpu, oracle): {detail}"


def test_e2m1_stochastic_rounding_at_its_thresholds():
    rng = np.random.default_rng(11)
    xs, hs = [], []
    draws = np.array([0, 1, 2, 3, 255, 256, 4095, 32767, 32768, 32769, 65533, 65534, 65535], dtype=np.int64)
    draws = np.concatenate([draws, rng.integers(0, 1 << 16, 400)])
    for lo, hi in zip(E2M1[:-1], E2M1[1:]):
        step = hi - lo
        # the threshold lo + h 2^-16 step of each draw h is an exact fp32 value
        t = (np.float64(lo) + draws * 2.0 ** -16 * step).astype(np.float32)
        assert np.all(t.astype(np.float64) == np.float64(lo) + draws * 2.0 ** -16 * step)
        x = neighbours(t)
        h = np.tile(draws, 5)
        xs += [x, -x]
        hs += [h, h]
    # tiny magnitudes (round up only when the draw is 0), zeros, saturation, huge values
    special = np.array([0.0, 2.0 ** -149, 2.0 ** -126, 1e-30, 2.0 ** -18, 2.0 ** -17, 3 * 2.0 ** -18, 5.9999995, 6.0,
                        6.0000005, 7.9999995, 8.0, 11.5, 1e10, 2.0 ** 126], dtype=np.float32)
    for h in (0, 1, 2, 65535):
        xs += [special, -special]
        hs += [np.full(special.size, h), np.full(special.size, h)]
    # random magnitudes over the whole grid and below it
    r = (rng.uniform(-8, 8, 200_000) * 2.0 ** rng.integers(-12, 1, 200_000)).astype(np.float32)
    xs.append(r)
    hs.append(rng.integers(0, 1 << 16, r.size))
    x = np.concatenate(xs).astype(np.float32)
    h = np.concatenate(hs).astype(np.uint32)
    # the draw is the low half of the word; junk in the high half must not matter
    w = h | (rng.integers(0, 1 << 16, h.size).astype(np.uint32) << 16)
    got = run(Q.ROUND_E2M1_SR, x, w)
    want = np.array([O.e2m1_sr(float(a), float(b) * 2.0 ** -16) for a, b in zip(x, h)], dtype=np.uint8)
    check(got, want, x, w)


def test_e2m1_round_to_nearest_grid_and_ties():
    mids = np.array([(a + b) / 2 for a, b in zip(E2M1[:-1], E2M1[1:])] + E2M1 + [6.5, 7.0, 1e20], dtype=np.float32)
    x = neighbours(mids, 3)
    rng = np.random.default_rng(12)
    x = np.concatenate([x, -x, rng.uniform(-7, 7, 50_000).astype(np.float32)])
    got = run(Q.ROUND_E2M1_RN, x, None)
    want = np.array([O.e2m1_rtn(float(a)) for a in x], dtype=np.uint8)
    check(got, want, x, None)


def e4m3_values() -> np.ndarray:
    return np.array([O.e4m3_value(c) for c in range(0x7F)], dtype=np.float64)


def test_e4m3_round_to_nearest_every_code_and_midpoint():
    v = e4m3_values()
    pts = np.concatenate([v, (v[:-1] + v[1:]) / 2, [448.0, 460.0, 464.0, 480.0, 1e6]]).astype(np.float32)
    x = neighbours(pts[pts > 0], 2)
    x = np.concatenate([x, [0.0, 2.0 ** -149, 2.0 ** -12, 2.0 ** -11]]).astype(np.float32)
    got = run(Q.ROUND_E4M3_RN, x, None)
    want = np.array([O.e4m3_rne_sat(float(a)) for a in x], dtype=np.uint8)
    check(got, want, x, None)


def test_e4m3_stochastic_rounding_at_its_thresholds():
    """Thresholds lo + rho gap with rho = r 2^-24: for r a multiple of 16 they
    are exact fp32 values in every binade (a multiple of 8 in the subnormal
    range suffices), so the exact comparison is reached with equality."""
    v = e4m3_values()
    rng = np.random.default_rng(13)
    rs = np.concatenate([[0, 16, 32, 1 << 20, 1 << 23, (1 << 24) - 16], rng.integers(0, 1 << 20, 60) * 16])
    xs, ws = [], []
    for lo, hi in zip(v[:-1], v[1:]):
        t = (lo + rs * 2.0 ** -24 * (hi - lo)).astype(np.float32)
        assert np.all(t.astype(np.float64) == lo + rs * 2.0 ** -24 * (hi - lo))
        x = neighbours(t[t > 0], 1) if lo == 0 else neighbours(t, 1)
        r = np.tile(rs[t > 0] if lo == 0 else rs, 3)
        xs.append(x)
        ws.append((r.astype(np.uint32) << 8) | rng.integers(0, 256, r.size).astype(np.uint32))
    x = np.concatenate(xs + [np.array([0.0, 447.99997, 448.0, 449.0, 1e30], dtype=np.float32)])
    w = np.concatenate(ws + [rng.integers(0, 1 << 32, 5, dtype=np.uint64).astype(np.uint32)])
    r = rng.uniform(0, 460, 50_000).astype(np.float32) * (2.0 ** rng.integers(-14, 1, 50_000)).astype(np.float32)
    x = np.concatenate([x, r])
    w = np.concatenate([w, rng.integers(0, 1 << 32, r.size, dtype=np.uint64).astype(np.uint32)])
    got = run(Q.ROUND_E4M3_SR, x, w)
    want = np.array([O.e4m3_sr(float(a), float(b >> 8) * 2.0 ** -24) for a, b in zip(x, w)], dtype=np.uint8)
    check(got, want, x, w)


def test_e8m0_stochastic_rounding_at_its_thresholds():
    rng = np.random.default_rng(14)
    es = np.arange(-149, 128)
    rs = np.array([0, 2, 4, 1 << 22, 1 << 23, (1 << 24) - 2])
    xs, ws = [], []
    for r in rs:
        # 2^e (1 + r 2^-24) with r even is exact for normal 2^e; subnormal 2^e stay powers of two
        t = np.array([np.ldexp(1.0 + (r * 2.0 ** -24 if e >= -126 else 0.0), int(e)) for e in es[es < 127]],
                     dtype=np.float32)
        x = neighbours(t, 1)
        xs.append(x)
        ws.append(np.full(x.size, (int(r) << 8) | 0x5A, dtype=np.uint32))
    r = (rng.uniform(0.5, 2, 50_000) * 2.0 ** rng.integers(-140, 120, 50_000)).astype(np.float32)
    x = np.concatenate(xs + [r])
    w = np.concatenate(ws + [rng.integers(0, 1 << 32, r.size, dtype=np.uint64).astype(np.uint32)])
    keep = (x > 0) & np.isfinite(x)
    x, w = x[keep], w[keep]
    got = run(Q.ROUND_E8M0_SR, x, w)
    want = np.array([O.e8m0_sr(float(a), float(b >> 8) * 2.0 ** -24) for a, b in zip(x, w)], dtype=np.uint8)
    check(got, want, x, w)


def test_selftest_rounding_rejects_bad_arguments():
    x = torch.zeros(4, dtype=torch.float32, device="cuda")
    c = torch.empty(4, dtype=torch.uint8, device="cuda")
    s = ctypes_stream()
    L = Q.lib()
    assert L.qfp4_selftest_rounding(5, Q._ptr(x), Q._ptr(None), Q._ptr(c), 4, s) == Q.ERR_INVALID_ARG
    assert L.qfp4_selftest_rounding(-1, Q._ptr(x), Q._ptr(None), Q._ptr(c), 4, s) == Q.ERR_INVALID_ARG
    assert L.qfp4_selftest_rounding(Q.ROUND_E2M1_SR, Q._ptr(x), Q._ptr(None), Q._ptr(c), 4, s) == Q.ERR_INVALID_ARG
    assert L.qfp4_selftest_rounding(Q.ROUND_E2M1_RN, Q._ptr(x), Q._ptr(None), Q._ptr(c), -1, s) == Q.ERR_INVALID_ARG
    assert L.qfp4_selftest_rounding(Q.ROUND_E2M1_RN, Q._ptr(x), Q._ptr(None), Q._ptr(c), 0, s) == Q.OK


def ctypes_stream():
    return Q._stream(None)
