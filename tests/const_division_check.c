/* Property check of the constant-divisor division the CUDA quantizer uses for
 * the row scale (absmax / 127, (max - min) / 255, and 7, 15 for 4-bit codes).
 *
 * With y = RN(1/D), lo = RN(RN(1 - D*y) * y), q0 = RN(a*y + RN(a*lo)) and one
 * Markstein correction q = RN(q0 + RN(a - D*q0) * y), q must equal the IEEE
 * quotient RN(a/D) for every finite binary32 a other than -0 (where it gives
 * +0; the kernels never divide -0: an absmax is a maximum of absolute values
 * and max - min of equal values is +0 under round-to-nearest). It checks every
 * significand at the binade exponent fields given on the command line (the
 * whole range 0..254 was checked when the method was adopted). It prints y and
 * lo as hex so the caller can compare them with the kernel's literals.
 * Usage: const_division_check <exponent field>... ; exit status 0 iff exact. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

int main(int argc, char** argv) {
  static const int divisors[4] = {7, 15, 127, 255};
  long checked = 0, violations = 0;
  for (int di = 0; di < 4; ++di) {
    const float d = (float)divisors[di];
    const float y = 1.0f / d;
    const float lo = fmaf(-d, y, 1.0f) * y;
    printf("D=%d y=%a lo=%a\n", divisors[di], y, lo);
    for (int ai = 1; ai < argc; ++ai) {
      const uint32_t field = (uint32_t)atoi(argv[ai]);
      for (uint32_t m = 0; m < (1u << 23); ++m) {
        for (uint32_t sign = 0; sign < 2; ++sign) {
          const uint32_t bits = (sign << 31) | (field << 23) | m;
          if (bits == 0x80000000u) continue;  /* -0: outside the kernels' domain */
          float a;
          memcpy(&a, &bits, 4);
          const float want = a / d;
          const float q0 = fmaf(a, y, a * lo);
          const float got = fmaf(fmaf(-d, q0, a), y, q0);
          ++checked;
          if (memcmp(&want, &got, 4) != 0) {
            if (violations < 5) printf("violation: a=%a D=%d want=%a got=%a\n", a, divisors[di], want, got);
            ++violations;
          }
        }
      }
    }
  }
  printf("checked %ld values, %ld violations\n", checked, violations);
  return violations != 0;
}
