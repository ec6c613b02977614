"""CPU pins of the oracle's FP64 -> BF16 rounding (the FFN's hidden
activation is held in BF16 between its two linears; library reading).

The rounding is checked against brute force in exact rationals: the nearest
of all finite BF16 values, ties to the even bit pattern, overflow past the
midpoint above the largest finite value to infinity.
"""
import bisect
from fractions import Fraction

import numpy as np

import oracle

# every non-negative finite BF16 value, ascending (patterns 0x0000..0x7F7F)
_PATTERNS = np.arange(0x7F80, dtype=np.uint32)
_VALUES = (_PATTERNS << 16).view(np.float32).astype(np.float64)
_MAX = Fraction(float(_VALUES[-1]))
_HALF_ULP_TOP = Fraction(2) ** 119          # half the spacing just below 2^128


def brute_round(x: float) -> int:
    if x != x:
        return 0xFFC0 if np.signbit(x) else 0x7FC0
    sign = 0x8000 if np.signbit(x) else 0
    a = Fraction(abs(x)) if np.isfinite(x) else None
    if a is None or a >= _MAX + _HALF_ULP_TOP:
        return sign | 0x7F80
    i = bisect.bisect_left(_VALUES.tolist(), float(a))      # exact: doubles compare exactly
    if i < len(_VALUES) and Fraction(float(_VALUES[i])) == a:
        return sign | int(_PATTERNS[i])
    lo, hi = i - 1, i
    if hi >= len(_VALUES):                                    # between max and the overflow midpoint
        return sign | int(_PATTERNS[lo])
    dl = a - Fraction(float(_VALUES[lo]))
    dh = Fraction(float(_VALUES[hi])) - a
    if dl < dh or (dl == dh and _PATTERNS[lo] % 2 == 0):
        return sign | int(_PATTERNS[lo])
    return sign | int(_PATTERNS[hi])


def test_round_bf16_brute_force_random():
    rng = np.random.default_rng(71)
    n = 3000
    e = rng.integers(-140, 129, n)
    m = rng.uniform(0.5, 1.0, n)
    x = np.ldexp(m, e) * np.where(rng.random(n) < 0.5, -1.0, 1.0)
    got = oracle.round_bf16(x)
    for xi, gi in zip(x.tolist(), got.tolist()):
        assert gi == brute_round(xi), (xi, hex(gi), hex(brute_round(xi)))


def test_round_bf16_ties_go_to_even():
    rng = np.random.default_rng(72)
    pats = rng.integers(0x0001, 0x7F7E, 2000).astype(np.uint32)
    lo = (pats << 16).view(np.float32).astype(np.float64)
    hi = ((pats + 1) << 16).view(np.float32).astype(np.float64)
    mid = (lo + hi) / 2                                       # exact in double
    got = oracle.round_bf16(mid)
    want = np.where(pats % 2 == 0, pats, pats + 1).astype(np.uint16)
    assert np.array_equal(got, want)
    # one double-ulp either side of the midpoint decides by distance
    assert np.array_equal(oracle.round_bf16(np.nextafter(mid, 0)), pats.astype(np.uint16))
    assert np.array_equal(oracle.round_bf16(np.nextafter(mid, np.inf)), (pats + 1).astype(np.uint16))


def test_round_bf16_round_trips_every_value():
    got = oracle.round_bf16(_VALUES)
    assert np.array_equal(got, _PATTERNS.astype(np.uint16))
    assert np.array_equal(oracle.round_bf16(-_VALUES[1:]), (_PATTERNS[1:] | 0x8000).astype(np.uint16))


def test_round_bf16_special_values():
    big = float(_MAX + _HALF_ULP_TOP)
    cases = [
        (0.0, 0x0000), (-0.0, 0x8000), (np.inf, 0x7F80), (-np.inf, 0xFF80), (np.nan, 0x7FC0),
        (float(_MAX), 0x7F7F), (big, 0x7F80), (np.nextafter(big, 0), 0x7F7F), (1e300, 0x7F80),
        (2.0 ** -133, 0x0001), (2.0 ** -134, 0x0000), (1.5 * 2.0 ** -133, 0x0002), (3.0 * 2.0 ** -134, 0x0002),
        (2.0 ** -126, 0x0080), (1.0, 0x3F80), (1.0 + 2.0 ** -8, 0x3F80), (1.0 + 3 * 2.0 ** -8, 0x3F82),
    ]
    for x, want in cases:
        assert int(oracle.round_bf16(np.array([x]))[0]) == want, (x, want)
        assert brute_round(x) == want, x
