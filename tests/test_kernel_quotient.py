"""The quantizer kernels form x/s for BF16-valued x from the correctly rounded
reciprocal r = 1/s with one residual correction: q = x*r; e = fma(-q, s, x);
q = fma(e, r, q); sign of x (computed as q = fma(fma(q, s, -x), -r, q), which keeps the
sign of -0 by itself; the test checks the two forms agree bit for bit). This test proves, by exhaustive enumeration on the CPU,
that the E4M3 code of that quotient equals the code of the IEEE quotient x/s for every
BF16 amax (with s = fl32(amax/448) >= 2^-80; the kernels divide below that) and every
BF16 x with |x| <= amax. It checks the kernels' arithmetic identity only: it uses its
own brute-force E4M3 encoder and shares nothing with the oracle."""
import os
import subprocess
import tempfile

import pytest

SRC = r"""
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>
static float f_of(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t u_of(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
/* nearest E4M3 code by brute force over the 127 magnitudes, ties to even, saturating */
static int enc(float t) {
  int sign = signbit(t) ? 0x80 : 0;
  double a = fabs((double)t);
  if (a >= 448.0) return sign | 0x7E;
  int best = 0;
  double bd = 1e300;
  for (int c = 0; c < 127; ++c) {
    int e = (c >> 3) & 15, m = c & 7;
    double v = e ? ldexp(1.0 + m / 8.0, e - 7) : ldexp((double)m, -9);
    double d = fabs(v - a);
    if (d < bd || (d == bd && (c & 1) == 0)) { bd = d; best = c; }
  }
  return sign | best;
}
int main(void) {
  long long bad = 0, total = 0;
#pragma omp parallel for reduction(+ : bad, total) schedule(dynamic, 64)
  for (uint32_t ab = 1; ab < 0x7F80; ++ab) {
    float amax = f_of(ab << 16);
    volatile float s = amax / 448.0f;
    if (s < 0x1p-80f) continue;
    volatile float r = 1.0f / s;
    for (uint32_t xb = 0; xb < 0x10000; ++xb) {
      if ((xb & 0x7FFF) > ab) continue;
      float x = f_of(xb << 16);
      volatile float t = x / s;
      float q = x * r;
      float e = fmaf(-q, s, x);
      float q2 = copysignf(fmaf(e, r, q), x);
      /* the kernels' sign-preserving form: q*s - x and q - (q*s - x)*r keep the sign of
         x = -0 without a copy-sign; it must equal q2 bit for bit */
      float en = fmaf(q, s, -x);
      float q3 = fmaf(en, -r, q);
      if (u_of(q3) != u_of(q2)) bad++;
      total++;
      if (u_of(q2) != u_of(t)) {
        if (fabsf(t) >= 0x1p-11f || fabsf(q2) >= 0x1p-11f) {
          if (enc(q2) != enc(t)) bad++;
        } else if (signbit(q2) != signbit(t)) {
          bad++;  /* below 2^-11 both encode to a signed zero */
        }
      }
    }
  }
  printf("%lld %lld\n", total, bad);
  return bad != 0;
}
"""


def test_reciprocal_quotient_gives_ieee_codes_exhaustively():
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "q.c")
        exe = os.path.join(d, "q")
        open(c, "w").write(SRC)
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                               c, "-o", exe, "-lm"])
        out = subprocess.run([exe], capture_output=True, text=True, timeout=900)
        total, bad = map(int, out.stdout.split())
        assert total > 10 ** 9
        assert bad == 0 and out.returncode == 0

