/* Check of the per-tensor quantizer's bracketing scheme (host restatement,
 * IEEE binary32 round-to-nearest-even, no flush-to-zero).
 *
 * The per-tensor delayed-scaling quantizer needs code(RN(x / s)), where code
 * is the saturating round-to-nearest-even conversion to E4M3 or E5M2 and s
 * is an arbitrary positive scale.  Instead of a division per element it
 * takes y = RN(1 / s) once, then
 *     y_lo = RN(y * (1 - 2^-20)),  y_hi = RN(y * (1 + 2^-20))
 * and per element c_lo = code(RN(x * y_lo)), c_hi = code(RN(x * y_hi)); if
 * c_lo == c_hi that is the code, otherwise it divides.  For s in
 * [2^-125, 2^125], y_lo < 1/s < y_hi as real numbers (|y - 1/s| <= 2^-24 / s,
 * and the factor 1 -+ 2^-20 moves y by far more than the two roundings), so
 * x * y_lo, x / s, x * y_hi are ordered (reversed for x < 0); RN and code
 * are monotone, so equal codes at both ends force the same code in between,
 * over the whole range (underflow, overflow, signed zeros).  Outside that
 * range of s the quantizer sets y_lo = 0 and y_hi = +inf, which makes the
 * two codes differ for every non-NaN x and so always divides.  This is the
 * rounding test of A. Ziv, "Fast evaluation of elementary mathematical
 * functions with correctly rounded last bit", ACM TOMS 17(3), 1991, applied
 * to one division.
 *
 * Checked here for every bf16 x (both signs) against s = RN(h / Q) for every
 * positive finite bf16 h (the history values the quantizer itself writes)
 * and for 4000 seeded random scales spread over all binades plus the edges
 * of the fast range: the scheme's code equals code(RN(x / s)) every time.
 * Argument: Q = 448 (E4M3, the default) or 57344 (E5M2).
 * Prints "pairs <n> bad <a> slow <b>"; exit status 0 iff a == 0.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* Saturating round-to-nearest-even onto the E4M3 (mbits 3, bias 7, max 448)
 * or E5M2 (mbits 2, bias 15, max 57344) grid; NaN -> sign | 0x7F. */
static int encode(float v, int e5m2) {
  const int mbits = e5m2 ? 2 : 3, emin = e5m2 ? -14 : -6, bias = e5m2 ? 15 : 7;
  const float qmax = e5m2 ? 57344.0f : 448.0f;
  const int sign = (to_bits(v) >> 31) ? 0x80 : 0;
  const float a = fabsf(v);
  if (isnan(v)) return sign | 0x7F;
  if (a >= qmax) return sign | (e5m2 ? 0x7B : 0x7E);
  int e;
  frexpf(a, &e);
  e -= 1; /* a in [2^e, 2^(e+1)) for a > 0 */
  if (a == 0.0f || e < emin) {
    const float k = nearbyintf(ldexpf(a, mbits - emin)); /* subnormal grid */
    return sign | (int)k;
  }
  const float k = nearbyintf(ldexpf(a, mbits - e)); /* in [2^mbits, 2^(mbits+1)] */
  return sign | ((e + bias) << mbits) + ((int)k - (1 << mbits));
}

static uint64_t rng = 0x9E3779B97F4A7C15ull;
static uint32_t next32(void) {
  rng ^= rng << 13; rng ^= rng >> 7; rng ^= rng << 17;
  return (uint32_t)(rng >> 16);
}

int main(int argc, char** argv) {
  const float qmax = argc > 1 ? (float)atof(argv[1]) : 448.0f;
  const int e5m2 = qmax > 448.0f;
  enum { kRandom = 4000, kEdges = 8 };
  const int nh = 0x7F80 - 1;
  const int nscale = nh + kRandom + kEdges;
  float* scales = (float*)malloc(sizeof(float) * nscale);
  for (int i = 0; i < nh; ++i) scales[i] = from_bits((uint32_t)(i + 1) << 16) / qmax;
  for (int i = 0; i < kRandom; ++i) {
    uint32_t b;
    do { b = next32() & 0x7FFFFFFFu; } while (b == 0 || b >= 0x7F800000u);
    scales[nh + i] = from_bits(b);
  }
  const float edges[kEdges] = {0x1p-125f, 0x1p125f, nextafterf(0x1p-125f, 0.0f), nextafterf(0x1p125f, INFINITY),
                               0x1p-149f, 0x1.fffffep127f, 1.0f, nextafterf(1.0f, 0.0f)};
  for (int i = 0; i < kEdges; ++i) scales[nh + kRandom + i] = edges[i];

  long long pairs = 0, bad = 0, slow = 0;
#pragma omp parallel for schedule(dynamic, 16) reduction(+ : pairs, bad, slow)
  for (int si = 0; si < nscale; ++si) {
    const float s = scales[si];
    float ylo = 0.0f, yhi = INFINITY;
    if (s >= 0x1p-125f && s <= 0x1p125f) {
      const float y = 1.0f / s;
      ylo = y * (1.0f - 0x1p-20f);
      yhi = y * (1.0f + 0x1p-20f);
    }
    for (uint32_t xb = 0; xb < 0x10000u; ++xb) {
      const float x = from_bits(xb << 16);
      if (isnan(x)) continue;
      const int ref = encode(x / s, e5m2);
      const int lo = encode(x * ylo, e5m2), hi = encode(x * yhi, e5m2);
      ++pairs;
      if (lo == hi) {
        if (lo != ref) ++bad;
      } else {
        ++slow;
      }
    }
  }
  printf("pairs %lld bad %lld slow %lld\n", pairs, bad, slow);
  free(scales);
  return bad == 0 ? 0 : 1;
}
