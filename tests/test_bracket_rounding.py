"""The quantiser's bracketed roundings, checked on the CPU in exact float32
arithmetic against the correctly rounded divisions the method defines.

The GPU quantiser does not divide per element: it multiplies by an
approximate reciprocal r of the divisor, scaled by 1 - 2^-20 and by
1 + 2^-20, and takes the code only where both products round to the same
code (else it falls back to the correctly rounded division).  That is exact
if the two products always lie below and above the correctly rounded
quotient, for any reciprocal within the stated error, because E2M1 and E4M3
rounding are monotone.  These tests emulate the products with the worst
reciprocal errors allowed (one ulp either way for the approximate
reciprocal, two for the scale step's 1/(6 G)) on inputs crowded at every
rounding threshold, and check that no agreeing bracket ever yields a code
different from the exact one.
"""
import numpy as np

from oracle import formats as F

f32 = np.float32
LO, HI = f32(1 - 2.0 ** -20), f32(1 + 2.0 ** -20)
E2M1_THRESHOLDS = np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])


def _perturbed(r, ulps):
    """r moved by `ulps` units in the last place (float32)."""
    r = np.asarray(r, f32)
    step = np.spacing(r)
    return (r.astype(np.float64) + ulps * step.astype(np.float64)).astype(f32)


def test_element_bracket_never_disagrees_with_exact_division():
    rng = np.random.default_rng(31)
    n = 60_000
    checked = agreed = 0
    for _ in range(4):
        d = (rng.uniform(0.5, 1.0, n) * 2.0 ** rng.integers(-40, 12, n)).astype(f32)
        # quotients on and next to every threshold (and at random), both signs
        t = np.concatenate([E2M1_THRESHOLDS, np.float32([0.0, 0.3, 6.0, 6.3])])[rng.integers(0, 11, n)]
        ulp_off = rng.integers(-6, 7, n)
        q = _perturbed(t, ulp_off).astype(np.float64) * rng.choice([-1.0, 1.0], n)
        w = F.bf16_to_f32(F.f64_to_bf16_rne(q * d.astype(np.float64)))
        exact = F.e2m1_encode((w / d).astype(f32))      # numpy float32 division is correctly rounded
        for ulps in (-1, 0, 1):                          # the reciprocal's allowed error
            r = _perturbed((f32(1) / d).astype(f32), ulps)
            lo = F.e2m1_encode((w * (r * LO).astype(f32)).astype(f32))
            hi = F.e2m1_encode((w * (r * HI).astype(f32)).astype(f32))
            same = lo == hi
            checked += n
            agreed += int(np.count_nonzero(same))
            assert np.array_equal(lo[same], exact[same])
    # the bracket decides almost everything; the rest takes the exact division
    assert agreed > 0.99 * checked


def test_scale_bracket_never_disagrees_with_exact_division():
    rng = np.random.default_rng(32)
    n = 60_000
    checked = agreed = 0
    for _ in range(4):
        amax = F.bf16_to_f32(F.f64_to_bf16_rne(rng.uniform(0.01, 100, n) * 2.0 ** rng.integers(-30, 30, n)))
        G = (amax / f32(2688)).astype(f32)
        ab = F.bf16_to_f32(F.f64_to_bf16_rne(amax.astype(np.float64) * rng.uniform(0, 1, n)))
        exact = F.e4m3_encode_satfinite(((ab / f32(6)).astype(f32) / G).astype(f32))
        g6 = (f32(6) * G).astype(f32)
        for ulps in (-2, 0, 2):                         # 1 / (6 G): two roundings
            k = _perturbed((f32(1) / g6).astype(f32), ulps)
            lo = F.e4m3_encode_satfinite((ab * (k * LO).astype(f32)).astype(f32))
            hi = F.e4m3_encode_satfinite((ab * (k * HI).astype(f32)).astype(f32))
            same = lo == hi
            checked += n
            agreed += int(np.count_nonzero(same))
            assert np.array_equal(lo[same], exact[same])
    assert agreed > 0.98 * checked


def test_bracket_detects_a_planted_threshold_hit():
    """A quotient exactly on a threshold whose tie goes up (0.75 -> 1.0) with
    the lower bracket end below it: the two ends must disagree, so the
    exact division decides."""
    d = f32(1.0)
    w = f32(0.75)
    r = _perturbed(f32(1) / d, -1)
    lo = F.e2m1_encode(np.float32([w * f32(r * LO)]))
    hi = F.e2m1_encode(np.float32([w * f32(r * HI)]))
    assert lo[0] != hi[0]
    assert F.e2m1_encode(np.float32([w / d]))[0] == hi[0]
