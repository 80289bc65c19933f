"""Pins of the oracle's quantisers and its FP16 rounding, against things other
than their own formulas: numpy's binary16 conversion, brute-force searches,
enumeration of every code, and round-trip identities.

Readings (the pages fix only the formats): Q1_0_g128 takes sign = (w >= 0)
and the group's mean |w| as scale ("Bonsai-27B-gguf technical white paper
digest", "technical architecture highlights"); INT4_G64 is symmetric
round-to-nearest with d = max|w| / 7 ("acorn-llm 0.11.4", "int4 quantisation
quality: group quantisation")."""
import numpy as np
import pytest

import oracle


def f16(bits) -> float:
    return float(np.array([bits], np.uint16).view(np.float16)[0])


# ---------------------------------------------------------------------------
# FP16 rounding: nearest, ties to even, saturating at 65504
# ---------------------------------------------------------------------------

def test_f16_every_finite_half_maps_to_itself():
    for h in range(0x10000):
        if (h & 0x7C00) == 0x7C00:
            continue  # inf / NaN
        assert oracle.f64_to_f16(f16(h)) == h, hex(h)


def test_f16_matches_numpy_rounding():
    g = np.random.default_rng(7)
    mant = g.uniform(0.5, 1.0, 20000)
    exp = g.integers(-30, 17, 20000)
    v = np.ldexp(mant, exp) * np.where(g.random(20000) < 0.5, -1.0, 1.0)
    v = v[np.abs(v) < 65504.0]
    want = v.astype(np.float16).view(np.uint16)  # numpy: nearest, ties to even
    got = np.array([oracle.f64_to_f16(x) for x in v], np.uint16)
    assert np.array_equal(got, want)


def test_f16_midpoints_round_to_even():
    # the exact midpoint between neighbouring positive halves goes to the one
    # with the even last mantissa bit; a hair above goes up, below goes down
    g = np.random.default_rng(8)
    for h in g.integers(1, 0x7BFF, 3000):
        lo, hi = f16(int(h)), f16(int(h) + 1)
        mid = (lo + hi) / 2.0
        even = int(h) if (int(h) & 1) == 0 else int(h) + 1
        assert oracle.f64_to_f16(mid) == even
        assert oracle.f64_to_f16(np.nextafter(mid, np.inf)) == int(h) + 1
        assert oracle.f64_to_f16(np.nextafter(mid, -np.inf)) == int(h)


def test_f16_saturation_and_specials():
    assert oracle.f64_to_f16(65504.0) == 0x7BFF
    assert oracle.f64_to_f16(65519.9) == 0x7BFF
    assert oracle.f64_to_f16(1e30) == 0x7BFF
    assert oracle.f64_to_f16(-1e30) == 0xFBFF
    assert oracle.f64_to_f16(0.0) == 0x0000
    assert oracle.f64_to_f16(-0.0) == 0x8000
    assert oracle.f64_to_f16(float("nan")) == 0
    assert oracle.f64_to_f16(2.0 ** -24) == 0x0001        # smallest subnormal
    assert oracle.f64_to_f16(2.0 ** -25) == 0x0000        # tie to even (zero)
    assert oracle.f64_to_f16(3 * 2.0 ** -25) == 0x0002    # tie to even (2 quanta)


# ---------------------------------------------------------------------------
# Q1_0_g128 quantiser
# ---------------------------------------------------------------------------

def test_q1_scale_is_the_least_squares_scale():
    """Brute force: the d that minimises sum (w - d*sign(w))^2 over a fine grid
    is the oracle's scale, to within the grid step and FP16 rounding."""
    g = np.random.default_rng(11)
    w = (g.standard_normal((6, 256)) * g.uniform(0.01, 3.0, (6, 1))).astype(np.float32)
    codes, scales = oracle.q1_quantize(w)
    s = np.where(codes == 1, 1.0, -1.0)
    for n in range(6):
        for grp in range(2):
            wg = w[n, 128 * grp:128 * (grp + 1)].astype(np.float64)
            sg = s[n, 128 * grp:128 * (grp + 1)]
            top = 2.0 * np.abs(wg).max()
            grid = np.linspace(0.0, top, 200001)
            sse = ((wg[None, :] - grid[:, None] * sg[None, :]) ** 2).sum(axis=1)
            best = grid[np.argmin(sse)]
            d = f16(int(scales[n, grp]))
            assert abs(d - best) <= top / 200000 + abs(best) * 2.0 ** -11


def test_q1_signs_and_special_values():
    w = np.zeros((1, 128), np.float32)
    w[0, :4] = [1.5, -2.0, -0.0, np.nan]
    w[0, 4:8] = [np.inf, -np.inf, 1e-30, -1e-30]
    codes, scales = oracle.q1_quantize(np.where(np.isfinite(w), w, 0).astype(np.float32))
    assert list(codes[0, :8]) == [1, 0, 1, 1, 1, 1, 1, 0]
    codes, _ = oracle.q1_quantize(w)
    assert list(codes[0, :8]) == [1, 0, 1, 0, 1, 0, 1, 0]  # -0.0 -> +1, NaN -> -1
    z, zs = oracle.q1_quantize(np.zeros((2, 256), np.float32))
    assert (z == 1).all() and (zs == 0).all()


def test_q1_round_trip_is_identity():
    """Weights that are already sign * fp16 scale quantise back to themselves."""
    g = np.random.default_rng(12)
    codes = g.integers(0, 2, (5, 384)).astype(np.int8)
    sbits = (np.abs(g.standard_normal((5, 3)) * 0.02).astype(np.float16)).view(np.uint16)
    sbits[sbits == 0] = 0x1400
    d = sbits.view(np.float16).astype(np.float32)
    w = np.where(codes == 1, 1.0, -1.0).astype(np.float32) * np.repeat(d, 128, axis=1)
    c2, s2 = oracle.q1_quantize(w)
    assert np.array_equal(c2, codes) and np.array_equal(s2, sbits)


# ---------------------------------------------------------------------------
# INT4_G64 quantiser
# ---------------------------------------------------------------------------

def test_int4_codes_are_the_nearest_of_all_sixteen():
    """Enumerate every code: q is the nearest of -8..7 times the stored scale
    (ties to the even code), and the scale is fp16(max|w| / 7)."""
    g = np.random.default_rng(13)
    w = (g.standard_normal((4, 256)) * 0.3).astype(np.float32)
    codes, scales = oracle.int4_quantize(w)
    allq = np.arange(-8, 8)
    for n in range(4):
        for grp in range(4):
            wg = w[n, 64 * grp:64 * (grp + 1)].astype(np.float64)
            d = f16(int(scales[n, grp]))
            assert scales[n, grp] == np.float16(np.abs(wg).max() / 7.0).view(np.uint16)
            for k in range(64):
                err = np.abs(wg[k] - allq * d)
                best = allq[err == err.min()]
                want = best[0] if len(best) == 1 else best[(best % 2) == 0][0]
                assert codes[n, 64 * grp + k] == want
    assert codes.min() >= -7 and codes.max() <= 7


def test_int4_round_trip_is_identity():
    """q * d with a +-7 in every group quantises back to (q, d)."""
    g = np.random.default_rng(14)
    q = g.integers(-7, 8, (6, 256)).astype(np.int8)
    for grp in range(4):
        q[:, 64 * grp + g.integers(0, 64)] = np.where(g.random(6) < 0.5, 7, -7)
    sbits = (np.abs(g.standard_normal((6, 4)) * 0.01).astype(np.float16)).view(np.uint16)
    sbits[sbits == 0] = 0x1400
    d = sbits.view(np.float16).astype(np.float32)
    w = q.astype(np.float32) * np.repeat(d, 64, axis=1)
    c2, s2 = oracle.int4_quantize(w)
    assert np.array_equal(c2, q) and np.array_equal(s2, sbits)


def test_int4_zero_and_nan_groups():
    w = np.zeros((1, 128), np.float32)
    w[0, 64:] = 1.0
    w[0, 70] = np.nan
    codes, scales = oracle.int4_quantize(w)
    assert (codes[0, :64] == 0).all() and scales[0, 0] == 0
    assert codes[0, 70] == 0 and (np.delete(codes[0, 64:], 6) == 7).all()


# ---------------------------------------------------------------------------
# properties over random inputs (hypothesis)
# ---------------------------------------------------------------------------

from hypothesis import given, settings, strategies as st  # noqa: E402

_floats = st.floats(min_value=-1e4, max_value=1e4, allow_nan=False, allow_infinity=False, width=32)


def _sse(w, s, d):
    return float(((w - d * s) ** 2).sum())


@settings(max_examples=60, deadline=None)
@given(st.lists(_floats, min_size=128, max_size=128))
def test_q1_scale_beats_its_fp16_neighbours(vals):
    """The squared error is a convex quadratic in d, so the fp16 scale the
    oracle picks must do at least as well as the neighbouring fp16 values."""
    w = np.array(vals, np.float32)[None, :]
    codes, scales = oracle.q1_quantize(w)
    s = np.where(codes[0] == 1, 1.0, -1.0)
    wd = w[0].astype(np.float64)
    h = int(scales[0, 0])
    best = _sse(wd, s, f16(h))
    for nb in (h - 1, h + 1):
        if 0 <= nb <= 0x7BFF:
            assert best <= _sse(wd, s, f16(nb)) * (1 + 1e-12) + 1e-300


@settings(max_examples=60, deadline=None)
@given(st.lists(_floats, min_size=64, max_size=64))
def test_int4_codes_are_nearest_for_their_scale(vals):
    w = np.array(vals, np.float32)[None, :]
    codes, scales = oracle.int4_quantize(w)
    d = f16(int(scales[0, 0]))
    wd = w[0].astype(np.float64)
    allq = np.arange(-8, 8)
    for k in range(64):
        err = np.abs(wd[k] - allq * d).min()
        assert abs(wd[k] - codes[0, k] * d) <= err * (1 + 1e-12) + 1e-300
    assert codes.min() >= -7
