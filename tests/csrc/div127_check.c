/* Checks, with IEEE fp32 arithmetic on the host (the same correctly rounded
 * operations the GPU executes), that one Markstein correction step with the
 * constant c = RN(1/127),
 *     q0 = RN(a c),  e = RN(a - q0 127) (fused),  q = RN(q0 + e c) (fused),
 * returns the correctly rounded quotient a / 127 for every positive finite float
 * a whose bit pattern is a multiple of `stride` (stride 1: all 2^31 - 2^23 - 1 of
 * them). The reference is the double quotient rounded to float: a / 127 is never
 * within 2^-53 relative of a float midpoint, so that rounding is exact.
 * Prints "<checked> <wrong>". */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

int main(int argc, char** argv) {
  const uint32_t stride = argc > 1 ? (uint32_t)strtoul(argv[1], NULL, 10) : 1u;
  const float c = 1.0f / 127.0f;
  long wrong = 0, checked = 0;
  for (uint64_t u = stride; u < 0x7F800000u; u += stride) {
    const uint32_t bits = (uint32_t)u;
    float a;
    memcpy(&a, &bits, 4);
    const float ref = (float)((double)a / 127.0);
    const float q0 = a * c;
    const float e = fmaf(-q0, 127.0f, a);
    const float q = fmaf(e, c, q0);
    if (q != ref) {
      if (wrong < 5) fprintf(stderr, "mismatch at 0x%08x\n", bits);
      ++wrong;
    }
    ++checked;
  }
  printf("%ld %ld\n", checked, wrong);
  return 0;
}
