/* Checks the quotient scheme the rotate+quantize kernel uses against IEEE fp32
 * division: with rs = RN(1/s), q0 = RN(y rs), then twice e = y - q s (one fused
 * multiply-add) and q = RN(q + e rs) (fused), the result must equal RN(y / s).
 * Inputs: divisors over many binades and the absmax/127 scales the quantizer
 * produces; dividends random in [-127 s, 127 s] and clustered within a few ulps
 * of (n + 1/2) s, where rounding to an integer is decided.
 * Prints the number of mismatches and the number of cases. */
#include <math.h>
#include <stdlib.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static uint64_t st = 0x243F6A8885A308D3ull;
static uint64_t rnd(void) {
  st += 0x9E3779B97F4A7C15ull;
  uint64_t z = st;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
static float urand(void) { return (float)(rnd() >> 40) / (float)(1ull << 24); }

static float refine(float y, float s, float rs) {
  float q = y * rs;
  float e = fmaf(q, -s, y);
  q = fmaf(e, rs, q);
  e = fmaf(q, -s, y);
  q = fmaf(e, rs, q);
  return q;
}

static int same(float a, float b) {
  uint32_t ua, ub;
  memcpy(&ua, &a, 4);
  memcpy(&ub, &b, 4);
  return ua == ub;
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
      if (k % 2 == 0) {
        y = (2.0f * urand() - 1.0f) * 127.0f * s;
      } else {
        const int n = (int)(rnd() % 254) - 127;
        float t = ((float)n + 0.5f) * s;
        const int steps = (int)(rnd() % 9) - 4;
        for (int i = 0; i < (steps < 0 ? -steps : steps); ++i) t = nextafterf(t, steps < 0 ? -INFINITY : INFINITY);
        y = t;
      }
      const float want = y / s;
      const float got = refine(y, s, rs);
      ++cases;
      if (!same(want, got)) {
        if (bad < 5) fprintf(stderr, "mismatch y=%a s=%a want=%a got=%a\n", y, s, want, got);
        ++bad;
      }
    }
  }
  printf("%ld %ld\n", bad, cases);
  return 0;
}
