"""The FP8 requantizer (a8) divides arbitrary fp32 values x (a dequantized code times its
row scale) by a column scale s >= 2^-80, and forms that scale s = amax / 448 for
amax >= 2^-60, with the same residual correction as the other quantizers: y = fl32(1/s),
q = fl32(x y), t = q - fl32(q s - x) y, both steps fused multiply-adds. Markstein's theorem (y within half an ulp of 1/s, q within one ulp of
x/s, the residual exact) makes t the correctly rounded quotient fl32(x/s) whenever
nothing underflows; below that the E4M3 code is a signed zero either way.

This test checks the identity on the CPU in C (correctly rounded fmaf, no contraction):
over random operands of every magnitude the requantizer meets, and over quotients built
to sit as close to fp32 rounding midpoints as fp32 operands allow: the fp32 quotients
must agree bit for bit wherever x/s is a normal number, the E4M3 codes everywhere.
It checks the kernel's arithmetic identity only and shares nothing with the oracle."""
import os
import subprocess
import tempfile

SRC = r"""
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>
static float f_of(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t u_of(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static uint64_t st = 88172645463325252ull;
static uint64_t next(void) { st ^= st << 13; st ^= st >> 7; st ^= st << 17; return st; }
static double unif(void) { return (next() >> 11) * 0x1p-53; }
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
static long long total = 0, bad = 0;
static void check(float x, float s) {
  volatile float y = 1.0f / s;
  volatile float q = x * y;
  float en = fmaf(q, s, -x);
  float t = fmaf(en, -y, q);
  volatile float ref = x / s;
  total++;
  /* the fp32 quotient itself must agree wherever x/s is a normal number; below that
     (no longer covered by the theorem) only the codes must */
  if (u_of(t) != u_of(ref) && (fabsf(ref) >= 0x1p-126f || enc(t) != enc(ref))) bad++;
}
int main(void) {
  for (int i = 0; i < 4000000; ++i) {  /* random operands */
    float s = (float)ldexp(1.0 + unif(), (int)(next() % 141) - 80);
    float x = (float)((unif() * 2.0 - 1.0) * 448.0 * s);
    check(x, s);
    check(f_of(u_of(x) & 0xFFFFF000u), s);  /* short significands */
  }
  for (int i = 0; i < 4000000; ++i) {  /* quotients next to fp32 midpoints */
    float s = (float)ldexp(1.0 + unif(), (int)(next() % 141) - 80);
    float q = (float)ldexp(1.0 + unif(), (int)(next() % 30) - 21);
    double mid = ((double)q + (double)nextafterf(q, INFINITY)) / 2.0;
    float x = (float)(mid * (double)s);
    check(x, s);
    check(nextafterf(x, INFINITY), s);
    check(nextafterf(x, -INFINITY), s);
    check(-x, s);
  }
  for (int i = 0; i < 4000000; ++i) {  /* the column scale amax / 448, amax >= 2^-60 */
    float amax = (float)ldexp(1.0 + unif(), (int)(next() % 187) - 60);
    check(amax, 448.0f);
    check(f_of(u_of(amax) & 0xFFFF0000u), 448.0f);  /* BF16-valued amax */
  }
  for (int k = -40; k <= 40; ++k) {  /* tiny quotients, signed zeros */
    check((float)ldexp(1.0, k - 100), 0x1p-80f);
    check(-(float)ldexp(1.0, k - 100), 0x1p-79f);
  }
  check(-0.0f, 1.0f);
  check(0.0f, 0x1p-80f);
  printf("%lld %lld\n", total, bad);
  return bad != 0;
}
"""


def test_fma_quotient_is_the_ieee_quotient():
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "q.c")
        exe = os.path.join(d, "q")
        open(c, "w").write(SRC)
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", c, "-o", exe,
                               "-lm"])
        out = subprocess.run([exe], capture_output=True, text=True, timeout=900)
        total, bad = map(int, out.stdout.split())
        assert total > 3 * 10 ** 7
        assert bad == 0 and out.returncode == 0
