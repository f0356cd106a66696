/* Checks the oracle's fp32 e^t and silu(g) = g / (1 + e^-g) against the C
 * library's double-precision exp, for every fp32 argument in a range.
 *
 *   exp_silu_check <oracle.so> exp  <stride> [lo hi]   every stride-th float t in [lo, hi]
 *   exp_silu_check <oracle.so> silu <stride> [lo hi]   (defaults: [-20, 89] and [-100, 100])
 *
 * e^t: where the true value is at most FLT_MAX the result must be finite and
 * within 2 fp32 ulps of it; where it is above FLT_MAX the result must be +inf or
 * FLT_MAX (the value rounded within the ulp bound). silu: within 4 ulps of the
 * double value, with 2^-149 as the ulp of subnormal results, and never zero
 * where the double value rounds to a nonzero float.
 * Prints "<checked> <bad> <worst error in units of 1/1000 ulp>". */
#include <dlfcn.h>
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

typedef void (*array_fn)(const float*, int64_t, float*);

static double ulp_f32(double v) {
  const double a = fabs(v);
  if (a < ldexp(1.0, -126)) return ldexp(1.0, -149);
  int e;
  frexp(a, &e);           /* a = m 2^e, m in [0.5, 1) */
  if (e > 128) e = 128;
  return ldexp(1.0, e - 24);
}

static float from_bits(uint32_t u) {
  float f;
  memcpy(&f, &u, 4);
  return f;
}

static uint32_t to_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
}

/* The next stride-th bit patterns up to hi, as floats; *next is the cursor. */
static int64_t fill(uint32_t hi, uint32_t stride, float* buf, int64_t cap, uint64_t* next) {
  int64_t n = 0;
  while (*next <= hi && n < cap) {
    buf[n++] = from_bits((uint32_t)*next);
    *next += stride;
  }
  return n;
}

int main(int argc, char** argv) {
  if (argc < 4) return 2;
  void* h = dlopen(argv[1], RTLD_NOW);
  if (!h) { fprintf(stderr, "%s\n", dlerror()); return 2; }
  const int is_exp = strcmp(argv[2], "exp") == 0;
  array_fn fn = (array_fn)dlsym(h, is_exp ? "orc_exp_f32_array" : "orc_silu_f32_array");
  if (!fn) return 2;
  const uint32_t stride = (uint32_t)strtoul(argv[3], NULL, 10);

  const float lo = argc > 5 ? strtof(argv[4], NULL) : (is_exp ? -20.0f : -100.0f);
  const float hi_arg = argc > 5 ? strtof(argv[5], NULL) : (is_exp ? 89.0f : 100.0f);
  const int64_t cap = 1 << 24;
  float* in = malloc(sizeof(float) * cap);
  float* out = malloc(sizeof(float) * cap);
  long long checked = 0, bad = 0;
  double worst = 0.0;
  /* Bit patterns run upward from +0 to hi on the positive side and from -0 to lo
     on the negative side; each side starts at the range's end nearest zero. */
  for (int side = 0; side < 2; ++side) {
    uint64_t next;
    uint32_t hi;
    if (side == 0) {
      if (hi_arg < 0.0f) continue;
      next = lo > 0.0f ? to_bits(lo) : 0u;
      hi = to_bits(hi_arg);
    } else {
      if (lo >= 0.0f) continue;
      next = hi_arg < 0.0f ? to_bits(hi_arg) : 0x80000000u;
      hi = to_bits(lo);
    }
    for (;;) {
      const int64_t n = fill(hi, stride, in, cap, &next);
      if (n == 0) break;
      fn(in, n, out);
      long long b = 0;
      double w = 0.0;
#pragma omp parallel for reduction(+ : b) reduction(max : w) schedule(static)
      for (int64_t i = 0; i < n; ++i) {
        const double x = in[i];
        const double r = out[i];
        if (is_exp) {
          const double ref = exp(x);
          if (ref > FLT_MAX) {
            if (!(isinf(r) || r == FLT_MAX)) ++b;
            continue;
          }
          const double err = fabs(r - ref) / ulp_f32(ref);
          if (!isfinite(r) || err > 2.0) ++b;
          if (isfinite(r) && err > w) w = err;
        } else {
          const double ref = x / (1.0 + exp(-x));
          const double err = fabs(r - ref) / ulp_f32(ref);
          if (err > 4.0) ++b;
          if ((float)ref != 0.0f && r == 0.0) ++b;
          if (err > w) w = err;
        }
      }
      checked += n;
      bad += b;
      if (w > worst) worst = w;
    }
  }
  printf("%lld %lld %lld\n", checked, bad, (long long)(worst * 1000.0));
  free(in);
  free(out);
  return 0;
}
