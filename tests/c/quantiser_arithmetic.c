/* Checks of the two arithmetic identities the CUDA quantisers rely on, in
 * IEEE fp32 with fused multiply-add (fmaf), which the GPU's fp32 fma and
 * multiply match bit for bit. The oracle does not use them: it divides and
 * rounds the plain way.
 *
 * 1. Division by a constant d (7 and 127) from y = RN(1/d): q0 = RN(a*y),
 *    r = fma(-d, q0, a), q = fma(r, y, q0) equals RN(a/d).
 * 2. Nearest-even rounding of x/s for a bf16 x and an fp16 scale s through a
 *    snap to the 2^-13 grid: t = fma(x, r, 1536), c = (t + (1.5*2^23 - 1536))
 *    - 1.5*2^23 equals rint(x/s), for r = RN(1/s) moved by up to 4 ulps and
 *    |x| <= qmax * s.
 *
 * usage: quantiser_arithmetic STRIDE  (STRIDE = 1: exhaustive; larger values
 * sample every STRIDE-th fp32 numerator and fp16 scale). Prints the counts;
 * exit status 1 on any mismatch. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float f_of(uint32_t u) {
  float f;
  memcpy(&f, &u, 4);
  return f;
}

static uint32_t u_of(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
}

static float half_to_float(int h) {
  const int e = (h >> 10) & 31, m = h & 1023;
  return e == 0 ? ldexpf((float)m, -24) : ldexpf((float)(m | 1024), e - 25);
}

int main(int argc, char **argv) {
  const long stride = argc > 1 ? atol(argv[1]) : 1;
  long long n_div = 0, bad_div = 0, n_rnd = 0, bad_rnd = 0;
  const float ds[2] = {7.f, 127.f};
  for (int k = 0; k < 2; ++k) {
    const volatile float d = ds[k];
    const float y = 1.0f / d;
    /* every positive finite bf16 value, then a stride over all fp32 values */
    for (uint32_t b = 1; b < 0x7F80u; ++b) {
      const float a = f_of(b << 16);
      const float q = fmaf(fmaf(-d, a * y, a), y, a * y);
      ++n_div;
      if (q != a / d) ++bad_div;
    }
    for (uint64_t b = 1; b < 0x7F800000u; b += (uint64_t)stride * 4099u) {
      const float a = f_of((uint32_t)b);
      const float q = fmaf(fmaf(-d, a * y, a), y, a * y);
      ++n_div;
      if (q != a / d) ++bad_div;
    }
  }
  const float B = 12582912.f;
  const int perts[3] = {0, 4, -4};
  const float qmaxs[2] = {7.f, 127.f};
  for (int k = 0; k < 2; ++k) {
    for (int h = 1; h < 0x7C00; h += (int)stride) {
      const float s = half_to_float(h);
      for (int pi = 0; pi < 3; ++pi) {
        const float r = f_of(u_of(1.0f / s) + perts[pi]);
        for (uint32_t xb = 0; xb < 0x7F80u; ++xb) {
          const float x = f_of(xb << 16);
          if (x > qmaxs[k] * s) break;
          for (int sg = 0; sg < 2; ++sg) {
            const float xs = sg ? -x : x;
            const double ref = nearbyint((double)xs / (double)s);
            const float c = (fmaf(xs, r, 1536.f) + (B - 1536.f)) - B;
            ++n_rnd;
            if ((double)c != ref) ++bad_rnd;
          }
        }
      }
    }
  }
  printf("division: %lld checked, %lld mismatches\nrounding: %lld checked, %lld mismatches\n", n_div, bad_div, n_rnd,
         bad_rnd);
  return (bad_div || bad_rnd) ? 1 : 0;
}
