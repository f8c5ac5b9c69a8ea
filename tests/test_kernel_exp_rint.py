"""The SwiGLU kernel rounds l = x*log2(e) to an integer by adding 1.5 * 2^23 (for
|l| < 2^22 the sum's unit in the last place is 1, so the fp32 addition rounds l to the
nearest integer, ties to even) and reads the integer from the sum's low mantissa bits.
This test proves, for every fp32 l the clamped argument can produce (|l| <= 130), that
the shifted value minus the shift equals rint(l) and that the integer read from the
bits equals (int)rint(l). It checks the kernel's arithmetic identity only (C, on the
CPU), independent of the oracle."""
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
int main(void) {
  const float shift = 12582912.0f;  /* 1.5 * 2^23 */
  long long bad = 0, total = 0;
  const uint32_t lim = u_of(130.0f);
#pragma omp parallel for reduction(+ : bad, total) schedule(static, 1 << 16)
  for (int64_t i = 0; i <= (int64_t)lim; ++i) {
    for (int sgn = 0; sgn < 2; ++sgn) {
      float l = f_of((uint32_t)i | (sgn ? 0x80000000u : 0u));
      volatile float t = l + shift;
      volatile float n = t - shift;
      float r = rintf(l);
      int k = (int)(u_of(t) - u_of(shift));
      total++;
      if (u_of(n) != u_of(r) && !(n == 0.0f && r == 0.0f)) bad++;
      if (k != (int)r) bad++;
    }
  }
  printf("%lld %lld\n", total, bad);
  return bad != 0;
}
"""


def test_shift_rounding_equals_rint_for_all_clamped_arguments():
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "r.c")
        exe = os.path.join(d, "r")
        open(c, "w").write(SRC)
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                               c, "-o", exe, "-lm"])
        out = subprocess.run([exe], capture_output=True, text=True, timeout=900)
        total, bad = map(int, out.stdout.split())
        assert total > 2 * 10 ** 9
        assert bad == 0 and out.returncode == 0
