"""Host-side proofs behind the codec kernel's arithmetic (no GPU needed).

The codec stores per-token scales s = amax / 127 and amax / 7 rounded once in fp32
(the codec reading of the rit.work TriAttention page's 8-bit and 4-bit blocks). The
kernel forms them without a division, by Markstein's reciprocal-and-correction step:
q0 = RN(a r), e = RN(a - q0 b) (one fused multiply-add, exact residual), s = RN(q0 + e r)
with r = RN(1 / b). That equals RN(a / b) only for suitable (a, b); here it is checked
for every positive finite bf16 value a (amax is the magnitude of a bf16 input), in
exact rational arithmetic, for b = 127 and b = 7.
"""
from fractions import Fraction

import numpy as np


def rn32(x: Fraction) -> np.float32:
    """The fp32 nearest to x, ties to even."""
    c = np.float32(float(x))
    best = None
    for v in (c, np.nextafter(c, np.float32(np.inf)), np.nextafter(c, np.float32(-np.inf))):
        key = (abs(Fraction(float(v)) - x), int(np.float32(v).view(np.uint32)) & 1)
        if best is None or key < best[0]:
            best = (key, v)
    return np.float32(best[1])


def test_division_free_scale_is_the_ieee_quotient_for_every_bf16():
    vals = (np.arange(1, 0x7F80, dtype=np.uint32) << 16).view(np.float32)   # positive finite bf16
    for b in (127, 7):
        r = Fraction(float(rn32(Fraction(1, b))))
        bad = []
        for a in vals:
            A = Fraction(float(a))
            q0 = Fraction(float(rn32(A * r)))
            e = Fraction(float(rn32(A - q0 * b)))
            if rn32(q0 + e * r) != rn32(A / b):
                bad.append(float(a))
        assert not bad, (b, bad[:5])
