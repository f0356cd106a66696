/* Checks the int8 code decision of the rotate+quantize kernel against its
 * definition, rne(RN(y / s)) with IEEE fp32 division. The kernel forms a
 * candidate n = rne(y rs) by one fused multiply-add onto 1.5 * 2^23
 * (rs = RN(1/s)), the residual r = RN(y - n s) by another, and accepts n when
 * |r| <= RN(s (1/2 - 2^-16)); otherwise it falls back to the correctly rounded
 * quotient (two Markstein steps) rounded half to even. Inputs: scales over many
 * binades and the absmax/127 scales the quantizer produces; dividends random in
 * [-127 s, 127 s], exact half-integer multiples (n + 1/2) s and values within a
 * few ulps of them.
 * Prints mismatches, cases and how many cases took the fallback. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static uint64_t st = 0x13198A2E03707344ull;
static uint64_t rnd(void) {
  st += 0x9E3779B97F4A7C15ull;
  uint64_t z = st;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
static float urand(void) { return (float)(rnd() >> 40) / (float)(1ull << 24); }

static long fallbacks = 0;

/* The residual bound's factor, 1/2 - 2^-16; a test builds this file with a
   looser factor to see that the check then reports mismatches. */
#ifndef BOUND
#define BOUND 0.4999847412109375f
#endif

static int code(float y, float s, float rs) {
  const float magic = 12582912.0f;
  const float t = s * BOUND;
  const float u = fmaf(y, rs, magic);
  const float n = u - magic;
  const float r = fmaf(n, -s, y);
  if (fabsf(r) <= t) return (int)n;
  ++fallbacks;
  float q = y * rs;
  float e = fmaf(q, -s, y);
  q = fmaf(e, rs, q);
  e = fmaf(q, -s, y);
  q = fmaf(e, rs, q);
  return (int)((q + magic) - magic);
}

int main(int argc, char** argv) {
  long n_div = argc > 1 ? atol(argv[1]) : 2000;
  long per = argc > 2 ? atol(argv[2]) : 20000;
  long bad = 0, cases = 0;
  for (long d = 0; d < n_div; ++d) {
    float s;
    if (d % 2 == 0) {
      float amax = ldexpf(1.0f + urand(), (int)(rnd() % 80) - 40);
      s = amax / 127.0f;
    } else {
      s = ldexpf(1.0f + urand(), (int)(rnd() % 160) - 80);
    }
    const float rs = 1.0f / s;
    for (long k = 0; k < per; ++k) {
      float y;
      if (k % 3 == 0) {
        y = (2.0f * urand() - 1.0f) * 127.0f * s;
      } else {
        const int n = (int)(rnd() % 254) - 127;
        float t = ((float)n + 0.5f) * s;
        const int steps = k % 3 == 1 ? 0 : (int)(rnd() % 9) - 4;
        for (int i = 0; i < (steps < 0 ? -steps : steps); ++i) t = nextafterf(t, steps < 0 ? -INFINITY : INFINITY);
        y = t;
      }
      const int want = (int)rintf(y / s);
      const int got = code(y, s, rs);
      ++cases;
      if (want != got) {
        if (bad < 5) fprintf(stderr, "mismatch y=%a s=%a want=%d got=%d\n", y, s, want, got);
        ++bad;
      }
    }
  }
  printf("%ld %ld %ld\n", bad, cases, fallbacks);
  return 0;
}
