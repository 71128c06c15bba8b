/* Property check of the division method the CUDA quantizer uses.
 *
 * With the two-term reciprocal y = RN(1/s), y_lo = RN(RN(1 - s*y) * y) (the
 * residual 1 - s*y is exact; it is checked here too), the first quotient
 * q0 = RN(v*y + RN(v*y_lo)) and one Markstein correction
 * q = RN(q0 + RN(v - s*q0) * y) (P. Markstein, IBM J. Res. Dev. 34(1), 1990),
 * the result must equal the IEEE quotient RN(v/s) whenever |v| >= 2^-100 and
 * s >= 2^-40 (the kernel's domain; smaller scales use the IEEE division).
 * Where |v| < 2^-100 a product or the remainder may underflow; there the true
 * quotient must be below 2^-60 in magnitude, and adding any offset with
 * 1/4 < |offset| < 2^20 must round the same way for both quotients (so no
 * code can change).
 * Samples: uniform quotients, quotients within a few ulps of half-integers and
 * of integers, large quotients, and random bit patterns. The host's binary32
 * division and fmaf are IEEE, as on the GPU.
 * Usage: division_method_check <samples> ; exit status 0 iff no violation. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static uint64_t st = 0x9E3779B97F4A7C15ull;
static uint64_t rnd(void) { st ^= st << 13; st ^= st >> 7; st ^= st << 17; return st; }
static float from_bits(uint32_t b) { float f; memcpy(&f, &b, 4); return f; }
static double unit(void) { return (double)(rnd() >> 11) / 9007199254740992.0; }
static float nudge(float v, int k) {
  for (; k > 0; --k) v = nextafterf(v, INFINITY);
  for (; k < 0; ++k) v = nextafterf(v, -INFINITY);
  return v;
}
static float quotient(float v, float s, float y, float y_lo) {
  const float q0 = fmaf(v, y, v * y_lo);
  const float r = fmaf(-s, q0, v);
  return fmaf(r, y, q0);
}

int main(int argc, char** argv) {
  const long n = argc > 1 ? atol(argv[1]) : 1000000L;
  long violations = 0, checked = 0, tiny = 0;
  for (long i = 0; i < n; ++i) {
    const float s = from_bits(((87u + (uint32_t)(rnd() % 140)) << 23) | (uint32_t)(rnd() & 0x7FFFFF));
    const float y = 1.0f / s;
    const float e = fmaf(-s, y, 1.0f);
    if ((double)e != 1.0 - (double)s * (double)y) {
      printf("violation: residual 1 - s*y not exact for s=%a\n", s);
      ++violations;
    }
    const float y_lo = e * y;
    float v;
    switch (rnd() % 5) {
      case 0: v = (float)((unit() * 512.0 - 256.0) * s); break;
      case 1: v = nudge((float)(((double)((int64_t)(rnd() % 512) - 256) + 0.5) * s), (int)(rnd() % 9) - 4); break;
      case 2: v = nudge((float)((double)((int64_t)(rnd() % 512) - 256) * s), (int)(rnd() % 9) - 4); break;
      case 3: v = nudge((float)(((double)((int64_t)(rnd() % (1ull << 31)) - (1ll << 30)) + 0.5) * s),
                        (int)(rnd() % 9) - 4); break;
      default:
        v = from_bits((uint32_t)rnd());
        if (!isfinite(v) || fabsf(v) > 256.0f * s) v = (float)((unit() - 0.5) * s);
    }
    if (!isfinite(v)) continue;
    ++checked;
    const float want = v / s;
    const float got = quotient(v, s, y, y_lo);
    if (memcmp(&want, &got, 4) == 0) continue;
    if (fabsf(v) >= 0x1p-100f) {
      if (violations < 5) printf("violation: v=%a s=%a want=%a got=%a\n", v, s, want, got);
      ++violations;
      continue;
    }
    ++tiny;
    if (!(fabsf(want) < 0x1p-60f)) {
      printf("violation: tiny v=%a gives quotient %a\n", v, want);
      ++violations;
      continue;
    }
    for (int t = 0; t < 8; ++t) {
      float off = (float)(0.25 + unit() * 1048575.75);
      if (rnd() & 1) off = -off;
      if (nearbyintf(want + off) != nearbyintf(got + off)) {
        printf("violation: offset %a flips a code (v=%a s=%a)\n", off, v, s);
        ++violations;
      }
    }
  }
  printf("checked %ld samples, %ld underflowing remainders, %ld violations\n", checked, tiny, violations);
  return violations != 0;
}
