/* Exhaustive checks of two short arithmetic sequences the decode kernel uses in place of
 * library division / reciprocal calls, each emulated here with IEEE single-precision
 * operations (fmaf and float multiplication round once, to nearest even):
 *
 *  div_q:  r = m / Q for Q in {7, 31, 127} as q0 = m * fl(1/Q); e = fma(-q0, Q, m);
 *          r = fma(e, fl(1/Q), q0). Checked against the correctly rounded quotient for every
 *          significand of m in [1, 2) and a spread of exponents.
 *  rcp16:  y = 1 / x for x an fp16 value (11-bit significand) as y0 = an approximation of
 *          1/x; y = fma(y0, fma(-x, y0, 1), y0). Checked against the correctly rounded
 *          reciprocal for every positive normal fp16 x, with y0 anywhere within 64 ulps of
 *          the true reciprocal (the hardware approximation is within one).
 *  rcp32:  y = 1 / x for any single-precision x (24-bit significand) as y0 = an approximation
 *          of 1/x, then two Newton steps in double precision, d = fma(d, fma(-x, d, 1), d)
 *          from d = y0, and one rounding of d to single precision. Checked against the
 *          correctly rounded reciprocal for every significand in [1, 2) at several exponents,
 *          with y0 at 0, +-1, +-2 and +-64 ulps from the true reciprocal.
 *
 * The references round an exact double-precision quotient to single precision; that equals the
 * correctly rounded single-precision quotient because m / Q (Q odd) and 1 / x (x with an
 * 11-bit significand) never lie within 2^-36 (relative) of a single-precision rounding
 * midpoint, far more than double precision's 2^-53, and 1 / x for a 24-bit significand x never
 * lies within 2^-49 of one (x times a 25-bit midpoint is never 1).
 *
 * Prints "div_mismatch=N rcp_mismatch=M cases=K". */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_of(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

static float f16_to_f32(uint16_t h) {  /* normal fp16 only */
  const uint32_t e = (h >> 10) & 31u, m = h & 1023u;
  return from_bits(((e - 15u + 127u) << 23) | (m << 13));
}

int main(void) {
  long long div_mis = 0, rcp_mis = 0, cases = 0;
  const int qs[3] = {7, 31, 127};
  const int exps[7] = {-14, -8, -1, 0, 1, 9, 15};
  for (int qi = 0; qi < 3; ++qi) {
    const float Q = (float)qs[qi];
    const float invQ = 1.0f / Q;
    for (int ei = 0; ei < 7; ++ei) {
      for (uint32_t s = 0; s < (1u << 23); ++s) {
        const float m = ldexpf(from_bits(0x3f800000u | s), exps[ei]);
        const float q0 = m * invQ;
        const float e = fmaf(-q0, Q, m);
        const float r = fmaf(e, invQ, q0);
        const float ref = (float)((double)m / (double)Q);
        cases++;
        if (bits_of(r) != bits_of(ref)) div_mis++;
      }
    }
  }
  for (uint32_t h = 0x0400u; h < 0x7c00u; ++h) {  /* positive normal fp16 */
    const float x = f16_to_f32((uint16_t)h);
    const float ref = (float)(1.0 / (double)x);
    for (int k = -64; k <= 64; ++k) {
      const float y0 = from_bits(bits_of(ref) + (uint32_t)k);
      const float y = fmaf(y0, fmaf(-x, y0, 1.0f), y0);
      cases++;
      if (bits_of(y) != bits_of(ref)) rcp_mis++;
    }
  }
  long long rcp32_mis = 0;
  const int rexps[5] = {-14, -3, 0, 6, 16};
  const int offs[7] = {0, 1, -1, 2, -2, 64, -64};
  for (int ei = 0; ei < 5; ++ei) {
    for (uint32_t s = 0; s < (1u << 23); ++s) {
      const float x = ldexpf(from_bits(0x3f800000u | s), rexps[ei]);
      const float ref = (float)(1.0 / (double)x);
      for (int k = 0; k < 7; ++k) {
        const float y0 = from_bits(bits_of(ref) + (uint32_t)offs[k]);
        double d = (double)y0;
        d = fma(d, fma(-(double)x, d, 1.0), d);
        d = fma(d, fma(-(double)x, d, 1.0), d);
        cases++;
        if (bits_of((float)d) != bits_of(ref)) rcp32_mis++;
      }
    }
  }
  printf("div_mismatch=%lld rcp_mismatch=%lld rcp32_mismatch=%lld cases=%lld\n", div_mis, rcp_mis,
         rcp32_mis, cases);
  return 0;
}
