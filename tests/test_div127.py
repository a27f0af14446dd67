"""The library reconstructs q / 127 for int8 codes q without a division
instruction: r = q * RN(1/127), e = q - 127 r (exact, by FMA), then
RN(r + e * RN(1/127)) (Markstein's correction).  This test proves, in exact
rational arithmetic, that the sequence returns the correctly rounded fp32
quotient for every one of the 256 codes, as IEEE division would."""
from fractions import Fraction

import numpy as np

f32 = np.float32


def _rn32(x: Fraction) -> float:
    """Round an exact rational to the nearest fp32, ties to even."""
    f = f32(float(x))  # within one ulp; fix up exactly below
    cands = [np.nextafter(f, f32(-np.inf)), f, np.nextafter(f, f32(np.inf))]

    def key(c):
        d = abs(Fraction(float(c)) - x)
        odd = int(np.array([c], dtype=np.float32).view(np.uint32)[0]) & 1
        return (d, odd)
    return float(min(cands, key=key))


def test_markstein_q_over_127_is_correctly_rounded_for_all_codes():
    inv = _rn32(Fraction(1, 127))
    for q in range(-128, 128):
        r = _rn32(Fraction(q) * Fraction(inv))
        e = _rn32(Fraction(q) - 127 * Fraction(r))          # fma(-r, 127, q): one rounding
        assert Fraction(e) == Fraction(q) - 127 * Fraction(r)  # and in fact exact
        out = _rn32(Fraction(e) * Fraction(inv) + Fraction(r))  # fma(e, inv, r)
        assert out == _rn32(Fraction(q, 127)), q
        assert out == float(f32(q) / f32(127))


def test_plain_multiply_would_not_be_exact():
    inv = f32(1) / f32(127)
    bad = [q for q in range(-128, 128) if f32(q) * inv != f32(q) / f32(127)]
    assert len(bad) > 0
