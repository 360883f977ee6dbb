/*
 * Test-side check of the oracle's E4M3 encoder over every fp32 bit pattern.
 *
 * An independent formulation of OCP FP8 E4M3 (bias 7, 3 mantissa bits,
 * largest finite 448, NaN = S.1111.111, no infinities) encoding with
 * round-to-nearest-even and saturation to +-448: the 127 non-negative finite
 * code values are built from the format definition, and a magnitude is
 * encoded as the NEAREST of them by binary search, a tie going to the even
 * code.  The oracle instead rounds arithmetically (exponent, quantum,
 * nearbyint); both must give the same byte for all 2^32 inputs.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

uint8_t orc_e4m3_from_float(float x);  /* the oracle's encoder (liboracle.so) */

static double g_val[127]; /* value of code c, c = 0 .. 126 (0x7E = 448) */

static void build_table(void) {
  for (int c = 0; c < 127; ++c) {
    const int e = c >> 3, m = c & 7;
    g_val[c] = e == 0 ? m * ldexp(1.0, -9) : (1.0 + m / 8.0) * ldexp(1.0, e - 7);
  }
}

static uint8_t nearest_code(float xf) {
  uint32_t bits;
  memcpy(&bits, &xf, 4);
  const uint8_t sign = (uint8_t)((bits >> 24) & 0x80);
  if (isnan(xf)) return (uint8_t)(sign | 0x7F);
  const double a = fabs((double)xf);
  if (a >= g_val[126]) return (uint8_t)(sign | 0x7E); /* saturate (infinities too) */
  int lo = 0, hi = 126;                                /* g_val[lo] <= a < g_val[hi] */
  while (hi - lo > 1) {
    const int mid = (lo + hi) / 2;
    if (g_val[mid] <= a) lo = mid; else hi = mid;
  }
  const double dl = a - g_val[lo], dh = g_val[hi] - a;
  int c;
  if (dl < dh) c = lo;
  else if (dh < dl) c = hi;
  else c = (lo & 1) == 0 ? lo : hi;                    /* tie: the even code */
  return (uint8_t)(sign | c);
}

/* Mismatches over the bit patterns [start, start + count); the first one in *first_bad. */
int64_t e4m3_mismatches(uint64_t start, uint64_t count, uint32_t* first_bad) {
  build_table();
  int64_t bad = 0;
  uint64_t first = UINT64_MAX;
#pragma omp parallel for reduction(+ : bad) reduction(min : first) schedule(static)
  for (int64_t i = 0; i < (int64_t)count; ++i) {
    const uint32_t b = (uint32_t)(start + (uint64_t)i);
    float x;
    memcpy(&x, &b, 4);
    if (orc_e4m3_from_float(x) != nearest_code(x)) {
      ++bad;
      if (b < first) first = b;
    }
  }
  if (first_bad) *first_bad = first == UINT64_MAX ? 0u : (uint32_t)first;
  return bad;
}
