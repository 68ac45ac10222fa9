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


# The codec's code quotients: q0 = RN(x r), e = RN(x - q0 s) (fused), q = RN(q0 + e r)
# with r = RN(1 / s), then rint(q), against rint(RN(x / s)) clamped to the plane's
# range (the oracle's IEEE division), for every pair of bf16 values 0 <= x <= amax
# (negative x follow by symmetry: every step rounds to nearest). C with fmaf and
# SSE single precision: IEEE binary32 operations, contraction off.
_QUOTIENT_CHECK = r"""
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>
static float f_of(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
int main(void) {
  const float lims[2] = {127.0f, 7.0f};
  for (int pl = 0; pl < 2; ++pl) {
    const float b = lims[pl];
    long long bad_fast = 0, bad_tiny = 0, checked = 0;
    float max_bad = 0.0f;
#pragma omp parallel for schedule(dynamic, 64) reduction(+ : bad_fast, bad_tiny, checked) reduction(max : max_bad)
    for (uint32_t ab = 1; ab < 0x7F80u; ++ab) {
      const float A = f_of(ab << 16);
      const float s = A / b;
      const float r = 1.0f / s;
      if (!(r < INFINITY)) continue;
      for (uint32_t xb = 0; xb <= ab; ++xb) {
        const float x = f_of(xb << 16);
        const float q0 = x * r;
        const float e = fmaf(-q0, s, x);
        const float q = fmaf(e, r, q0);
        float ref = rintf(x / s);
        if (ref > b) ref = b;
        ++checked;
        if (rintf(q) != ref) {
          if (A >= 0x1p-100f) ++bad_fast; else ++bad_tiny;
          if (A > max_bad) max_bad = A;
        }
      }
    }
    printf("%d %lld %lld %lld %a\n", (int)b, checked, bad_fast, bad_tiny, max_bad);
  }
  return 0;
}
"""


def test_division_free_codes_equal_the_ieee_quotient_codes(tmp_path):
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    assert gcc, "gcc is needed for this host check"
    src = tmp_path / "quotients.c"
    src.write_text(_QUOTIENT_CHECK)
    exe = tmp_path / "quotients"
    subprocess.run([gcc, "-O2", "-ffp-contract=off", "-fopenmp", str(src), "-o", str(exe), "-lm"], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    rows = [line.split() for line in out if line.strip()]
    assert [int(r[0]) for r in rows] == [127, 7]
    for lim, checked, bad_fast, bad_tiny, max_bad in rows:
        # every (x, amax) pair with a finite reciprocal scale was visited
        assert int(checked) > 5 * 10 ** 8
        # the kernel takes the division-free path only for amax >= 2^-100, where
        # it is exact; the few pairs it would get wrong lie far below (amax < 2^-117)
        assert int(bad_fast) == 0, (lim, bad_fast)
        assert float.fromhex(max_bad) < 2.0 ** -110, (lim, max_bad)


# The codec's reciprocal of a scale: a first guess r0 (the hardware approximation,
# documented within 1 ulp of 1/s), then e = RN(1 - s r0) and r = RN(r0 + e r0), both
# fused. For every scale s = RN(amax / b) of a bf16 row maximum amax >= 2^-100 (the
# division-free path) and every r0 within 3 ulps of RN(1/s), r must be RN(1/s).
_RECIPROCAL_CHECK = r"""
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>
static float f_of(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t u_of(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
int main(void) {
  const float lims[2] = {127.0f, 7.0f};
  for (int pl = 0; pl < 2; ++pl) {
    long long bad = 0, checked = 0;
    for (uint32_t ab = 1; ab < 0x7F80u; ++ab) {
      const float A = f_of(ab << 16);
      if (!(A >= 0x1p-100f)) continue;
      const float s = A / lims[pl];
      const float R = 1.0f / s;
      for (int k = -3; k <= 3; ++k) {
        const float r0 = f_of(u_of(R) + k);
        const float e = fmaf(-s, r0, 1.0f);
        ++checked;
        if (fmaf(e, r0, r0) != R) ++bad;
      }
    }
    printf("%d %lld %lld\n", (int)lims[pl], checked, bad);
  }
  return 0;
}
"""


def test_newton_step_gives_the_correctly_rounded_reciprocal_of_every_scale(tmp_path):
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    assert gcc, "gcc is needed for this host check"
    src = tmp_path / "reciprocal.c"
    src.write_text(_RECIPROCAL_CHECK)
    exe = tmp_path / "reciprocal"
    subprocess.run([gcc, "-O2", "-ffp-contract=off", str(src), "-o", str(exe), "-lm"], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    rows = [line.split() for line in out if line.strip()]
    assert [int(r[0]) for r in rows] == [127, 7]
    for lim, checked, bad in rows:
        assert int(checked) == 7 * 29184, (lim, checked)   # 29,184 maxima of bf16 in [2^-100, max]
        assert int(bad) == 0, (lim, bad)
