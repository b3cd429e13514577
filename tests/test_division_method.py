"""The quantizer divides by the group scale as q0 = RN(x r), e = x - q0 s
(one fma), q = RN(q0 + e r) with r = RN(1/s) (Markstein's correction step,
P. Markstein, IBM J. Res. Dev. 34(1), 1990), and relies on q being the IEEE
fp32 quotient x / s that the oracle computes.  x and s are fp16 values and no
step under- or overflows for them, so every step scales exactly with their
exponents and the identity only has to hold for every pair of 11-bit
significands: this test checks all 2047 x 2047 pairs (both signs of x) with
C's fp32 division and fmaf, which are correctly rounded.  The group scale
(max - min) / qmax divides an fp32 difference (any 24-bit significand) by
the constant qmax = 3, 15 or 255 with r = RN(1/qmax): checked for every
24-bit significand."""
import os
import shutil
import subprocess
import tempfile

import pytest

SRC = r"""
#include <math.h>
#include <stdio.h>
int main(void) {
  long bad = 0, n = 0;
  for (int S = 1; S < 2048; ++S) {
    volatile float s = (float)S;
    const float r = 1.0f / s;
    for (int X = -2047; X < 2048; ++X) {
      volatile float x = (float)X;
      const float q0 = x * r;
      const float e = fmaf(-q0, s, x);
      const float q = fmaf(e, r, q0);
      const float ref = x / s;
      ++n;
      if (q != ref) ++bad;
    }
  }
  long bad24 = 0, n24 = 0;
  const float qmax[3] = {3.0f, 15.0f, 255.0f};
  for (int k = 0; k < 3; ++k) {
    volatile float d = qmax[k];
    const float r = 1.0f / d;
    for (long m = 1L << 23; m < (1L << 24); ++m) {
      volatile float x = (float)m;
      const float q0 = x * r;
      const float e = fmaf(-q0, d, x);
      const float q = fmaf(e, r, q0);
      ++n24;
      if (q != x / d) ++bad24;
    }
  }
  printf("%ld %ld %ld %ld\n", n, bad, n24, bad24);
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_correction_step_equals_ieee_division_on_its_domains():
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "div.c")
        exe = os.path.join(d, "div")
        with open(c, "w") as f:
            f.write(SRC)
        subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-o", exe, c,
                        "-lm"], check=True)
        out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout.split()
    n, bad, n24, bad24 = (int(t) for t in out)
    assert n == 2047 * 4095 and n24 == 3 * (1 << 23)
    assert bad == 0
    assert bad24 == 0
