/* Exhaustive check of the scale division used by the row quantisers.
 *
 * The per-row scale is fl(m / 127) with m = max(row max |t|, 1e-8) (the
 * SmoothQuant page's per-token and per-channel quantisers divide the fp32
 * maximum by 127).  The kernels evaluate it without a division instruction:
 *     q0 = fl(m * r),  r = RN(1/127)
 *     e  = fma(-q0, 127, m)          (exact)
 *     q  = fma(e, r, q0)             (rounded once)
 * This program compares q with the IEEE quotient m / 127 for every positive
 * fp32 m from 1e-8 to the largest finite value and exits non-zero on any
 * difference.  Build with contraction off so that each step rounds as
 * written. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

int main(void) {
  const float b = 127.0f;
  const float r = (float)(1.0 / 127.0); /* RN(1/127): 1/127 is not a midpoint */
  float f = 1e-8f;
  uint32_t u, hi = 0x7F7FFFFFu;
  unsigned long long n = 0, bad = 0;
  memcpy(&u, &f, sizeof u);
  for (;; ++u) {
    float m, q0, e, q;
    memcpy(&m, &u, sizeof m);
    q0 = m * r;
    e = fmaf(-q0, b, m);
    q = fmaf(e, r, q0);
    if (q != m / b) {
      if (bad < 5) printf("m=%a: %a != %a\n", m, q, m / b);
      ++bad;
    }
    ++n;
    if (u == hi) break;
  }
  printf("%llu values, %llu differences\n", n, bad);
  return bad != 0;
}
