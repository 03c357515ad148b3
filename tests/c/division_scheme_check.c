/* Exhaustive check of the quantizers' division scheme (host restatement,
 * IEEE binary32 with fused multiply-add, no flush-to-zero).
 *
 * For a block with amax (a positive finite bf16 value) the FP32-mode scale is
 * s = RN(amax / 448).  The quantizer needs RN(x / s) for every bf16 x of the
 * block (|x| <= amax).  Instead of one division per element it takes the
 * reciprocal y = RN(1 / s) once and applies one Markstein correction step
 * (P. Markstein, IBM J. Res. Dev. 34(1), 1990) in its sign-symmetric form:
 *     q0 = RN(x * y);  r = fma(q0, s, -x);  q = fma(r, -y, q0)
 * (the same arithmetic as r = x - q0*s, q = q0 + r*y, up to the sign of an
 * exact zero, so that x = -0 gives q = -0).  Blocks with amax < 2^-80 divide.
 *
 * Claim checked here, over every positive finite bf16 amax >= 2^-80 and every
 * bf16 x (both signs) with |x| <= amax:
 *   (a) q == RN(x / s) bit for bit whenever |RN(x / s)| >= T or |q| >= T,
 *       T below half the format's smallest subnormal (the range where a
 *       code can be non-zero);
 *   (b) sign(q) == sign(RN(x / s)) always (signed-zero codes agree).
 * Argument: the format's largest value, 448 (E4M3, the default; T = 2^-12,
 * codes round to zero up to 2^-10) or 57344 (E5M2; T = 2^-17, codes round to
 * zero up to 2^-17: the tie at 2^-17 goes to the even code, zero).  In E5M2
 * terms the check is tight: the only differences below T sit at amax just
 * above 2^-80 with x near 2^-113, where the remainder is subnormal, and both
 * results encode to a signed zero.
 * Prints "pairs <n> bad <a> badsign <b>"; exit status 0 iff a == b == 0.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float from_bf16(uint32_t b) { uint32_t u = b << 16; float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

int main(int argc, char** argv) {
  const float qmax = argc > 1 ? (float)atof(argv[1]) : 448.0f;
  const float thr = qmax > 448.0f ? 0x1p-17f : 0x1p-12f;
  long long pairs = 0, bad = 0, badsign = 0;
#pragma omp parallel for schedule(dynamic, 64) reduction(+ : pairs, bad, badsign)
  for (uint32_t ab = 1; ab < 0x7F80u; ++ab) {
    const float amax = from_bf16(ab);
    if (!(amax >= 0x1p-80f)) continue;
    const float s = amax / qmax;
    const float y = 1.0f / s;
    for (uint32_t xb = 0; xb <= ab; ++xb) {
      for (int neg = 0; neg < 2; ++neg) {
        const float x = from_bf16(xb | (neg ? 0x8000u : 0u));
        const float ref = x / s;
        const float q0 = x * y;
        const float r = fmaf(q0, s, -x);
        const float q = fmaf(r, -y, q0);
        ++pairs;
        if (bits(q) != bits(ref) && (fabsf(ref) >= thr || fabsf(q) >= thr)) ++bad;
        if ((bits(q) ^ bits(ref)) & 0x80000000u) ++badsign;
      }
    }
  }
  printf("pairs %lld bad %lld badsign %lld\n", pairs, bad, badsign);
  return (bad == 0 && badsign == 0) ? 0 : 1;
}
