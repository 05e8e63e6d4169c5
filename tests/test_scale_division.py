"""The activation quantize computes scale = amax/448 as RN(amax*c) followed by one
FMA correction with the exact remainder (c = RN(1/448)), instead of an IEEE division.
This checks, with exact rational arithmetic, that the three roundings give the
correctly rounded quotient for every non-negative finite bf16 amax (the only
values amax can take), subnormals included."""
from fractions import Fraction

import numpy as np


def rn32(x: Fraction) -> np.float32:
    """Round an exact rational to the nearest float32, ties to even."""
    if x == 0:
        return np.float32(0.0)
    f = np.float32(float(x))
    cands = [np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))]
    return min(cands, key=lambda c: (abs(Fraction(float(c)) - x),
                                     int(np.array(c, dtype=np.float32).view(np.uint32)) & 1))


def test_fma_corrected_division_by_448_is_exact_for_every_bf16():
    c = np.float32(np.float32(1.0) / np.float32(448.0))
    C = Fraction(float(c))
    bits = (np.arange(0, 0x7F80, dtype=np.uint32) << 16).view(np.float32)
    bad = []
    for amax in bits:
        A = Fraction(float(amax))
        q0 = np.float32(amax * c)                       # one rounding, as numpy does in float32
        rem = rn32(A - Fraction(float(q0)) * 448)       # fma(-q0, 448, amax)
        s = rn32(Fraction(float(rem)) * C + Fraction(float(q0)))   # fma(rem, c, q0)
        if s != rn32(A / 448):
            bad.append(float(amax))
    assert not bad, bad[:5]
