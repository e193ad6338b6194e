/* Checks, against the host's IEEE division, the division-free fp32
 * quotients that the pack kernel uses on fp16 inputs (restated here from the
 * mathematics, independently of the kernel source):
 *
 *   scale:  s = RN(d / L), L = 15 or 3, for every fp32 d in [2^-24, 2^18)
 *           s = RN(d*yh + RN(d*yl)) with yh = RN(1/L), yl = RN(1/L - yh)
 *           (exhaustive over the range, so no correction step is needed)
 *   codes:  Q = RN(t / s) for t = RN(x - mn), s as above, x, mn, mx fp16
 *           (every fp16 x in [mn, mx] for many (mn, mx) pairs, including
 *           ranges that put t/s exactly on half-integers)
 *           yh = RN(1/s), yl = RN(RN(1 - s*yh)*yh),
 *           q0 = RN(t*yh + RN(t*yl)), Q = RN(q0 + RN(t - q0*s)*yh)
 *
 * The codes' quotient is Markstein's correction (a faithful first quotient,
 * an exact FMA remainder, one correction with the correctly rounded
 * reciprocal); the scale's first quotient needs none on its range.  fmaf is the correctly rounded fused multiply-add of C99.
 * Exit status 0 when every case matches. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float h2f(uint16_t h) {
  const uint32_t sgn = (uint32_t)(h & 0x8000u) << 16, e = (h >> 10) & 0x1fu, m = h & 0x3ffu;
  float f;
  if (e == 0) {
    f = ldexpf((float)m, -24);
    return sgn ? -f : f;
  }
  const uint32_t b = sgn | ((e + 112u) << 23) | (m << 13);
  memcpy(&f, &b, 4);
  return f;
}

static uint64_t state = 88172645463325252ull;
static uint64_t next(void) {
  state ^= state << 13;
  state ^= state >> 7;
  state ^= state << 17;
  return state;
}

static int cmpf(const void* a, const void* b) {
  const float x = *(const float*)a, y = *(const float*)b;
  return (x > y) - (x < y);
}

static float div_levels(float d, float L) {
  volatile float one = 1.0f;
  const float yh = one / L;
  const float yl = (float)(1.0 / (double)L - (double)yh);
  return fmaf(d, yh, d * yl);
}

int main(int argc, char** argv) {
  const long pairs = argc > 1 ? atol(argv[1]) : 4000;
  long bad = 0, checks = 0, ties = 0;
  /* scale: exhaustive over the range of max - min */
  const float Ls[2] = {15.0f, 3.0f};
  for (int k = 0; k < 2; ++k) {
    uint32_t lo, hi;
    float f = ldexpf(1.0f, -24);
    memcpy(&lo, &f, 4);
    f = ldexpf(1.0f, 18);
    memcpy(&hi, &f, 4);
    for (uint32_t b = lo; b < hi; ++b) {
      float d;
      memcpy(&d, &b, 4);
      volatile float want = d / Ls[k];
      ++checks;
      if (div_levels(d, Ls[k]) != want) ++bad;
    }
  }
  if (bad) {
    printf("scale: %ld mismatches\n", bad);
    return 1;
  }
  /* codes: all fp16 values inside sampled ranges */
  static float vals[65536];
  int nv = 0;
  for (uint32_t h = 0; h < 65536; ++h)
    if (((h >> 10) & 0x1f) != 0x1f) vals[nv++] = h2f((uint16_t)h);
  qsort(vals, nv, sizeof(float), cmpf);
  for (long p = 0; p < pairs; ++p) {
    int i = (int)(next() % nv), j = (int)(next() % nv);
    if (p % 4 == 1) j = i + (int)(next() % 64);
    if (p % 4 == 2) j = i + (int)(next() % 4096);
    if (p % 8 == 3) { /* range (levels) * odd * 2^e: exact half-integer quotients */
      const float lev = (next() & 1) ? 15.0f : 3.0f;
      const float d = lev * (float)(1 + 2 * (next() % 16)) * ldexpf(1.0f, (int)(next() % 30) - 22);
      const float target = vals[i] + d;
      int a = i, z = nv - 1;
      while (a < z) {
        const int mid = (a + z) / 2;
        if (vals[mid] < target) a = mid + 1; else z = mid;
      }
      j = a;
    }
    if (j >= nv) j = nv - 1;
    if (i > j) { const int t = i; i = j; j = t; }
    const float mn = vals[i], mx = vals[j];
    for (int b = 0; b < 2; ++b) {
      const float lev = b ? 3.0f : 15.0f;
      volatile float dd = mx - mn;
      float s = div_levels(dd, lev);
      if (mx == mn) s = 1.0f;
      volatile float one = 1.0f;
      const float yh = one / s;
      const float yl = fmaf(-s, yh, 1.0f) * yh;
      for (int k = i; k <= j; ++k) {
        volatile float t = vals[k] - mn;
        const float want = t / s;
        const float q0 = fmaf(t, yh, t * yl);
        const float q = fmaf(fmaf(-q0, s, t), yh, q0);
        ++checks;
        if (want - floorf(want) == 0.5f) ++ties;
        if (q != want) ++bad;
      }
    }
  }
  printf("checks %ld, exact half-integer quotients %ld, mismatches %ld\n", checks, ties, bad);
  return bad != 0;
}
