/*
 * IEEE-754 binary16 and bfloat16 rounding for the oracle (test
 * infrastructure only; see oref.h).
 *
 * Both conversions follow the definition directly: find the spacing q of the
 * destination format at |x| (the subnormal spacing below the smallest normal),
 * scale |x| to an integer count of q (an exact power-of-two scaling), round
 * that count to the nearest integer with ties to even, and re-encode. frexp and
 * ldexp only split or scale by powers of two, so every step is exact except the
 * one rounding the definition asks for.
 */
#include <math.h>
#include <string.h>

#include "oref.h"

/* Round a non-negative finite value v (an exact multiple of 2^-k for some k)
 * to the nearest integer, ties to even. */
static double round_half_even(double v) {
  double f = floor(v);
  double frac = v - f; /* exact: v and f share the exponent range */
  if (frac > 0.5) return f + 1.0;
  if (frac < 0.5) return f;
  return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* Generic RNE into a binary format with `mant` explicit mantissa bits,
 * exponent bias `bias` and `ebits` exponent bits. Returns the bit pattern
 * (without sign) of |x|; x must be finite. */
static uint32_t encode_rne(double ax, int mant, int bias, int ebits) {
  const int emin = 1 - bias;                 /* exponent of smallest normal */
  const int emax_field = (1 << ebits) - 1;   /* all-ones: inf / nan */
  if (ax == 0.0) return 0;
  int e;
  (void)frexp(ax, &e); /* ax = m * 2^e, m in [0.5, 1) -> unbiased exp e-1 */
  int E = e - 1;
  if (E < emin) E = emin; /* subnormal range uses the smallest normal spacing */
  /* spacing q = 2^(E - mant); count = ax / q */
  double count = ldexp(ax, mant - E);
  double r = round_half_even(count);
  /* r * 2^(E - mant) is the rounded magnitude; r may equal 2^(mant+1) */
  if (r >= ldexp(1.0, mant + 1)) { /* carried into the next binade */
    r = r / 2.0;
    E += 1;
  }
  if (r < ldexp(1.0, mant)) {
    /* subnormal (only possible when E == emin) or zero */
    return (uint32_t)r;
  }
  int field = E + bias;
  if (field >= emax_field) return (uint32_t)emax_field << mant; /* inf */
  uint32_t frac = (uint32_t)(r - ldexp(1.0, mant));
  return ((uint32_t)field << mant) | frac;
}

uint16_t oref_f64_to_f16(double x) {
  if (isnan(x)) return (uint16_t)(signbit(x) ? 0xFE00 : 0x7E00);
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  if (isinf(x)) return (uint16_t)(sign | 0x7C00);
  return (uint16_t)(sign | encode_rne(fabs(x), 10, 15, 5));
}

double oref_f16_to_f64(uint16_t h) {
  int sign = (h >> 15) & 1;
  int field = (h >> 10) & 0x1F;
  int frac = h & 0x3FF;
  double v;
  if (field == 0x1F) {
    v = frac ? NAN : INFINITY;
  } else if (field == 0) {
    v = ldexp((double)frac, -24);
  } else {
    v = ldexp((double)(frac | 0x400), field - 25);
  }
  return sign ? -v : v;
}

uint16_t oref_f64_to_bf16(double x) {
  if (isnan(x)) return (uint16_t)(signbit(x) ? 0xFFC0 : 0x7FC0);
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  if (isinf(x)) return (uint16_t)(sign | 0x7F80);
  return (uint16_t)(sign | encode_rne(fabs(x), 7, 127, 8));
}

uint16_t oref_f32_to_bf16(float x) { return oref_f64_to_bf16((double)x); }

double oref_bf16_to_f64(uint16_t b) {
  uint32_t bits = (uint32_t)b << 16;
  float f;
  memcpy(&f, &bits, sizeof f); /* bf16 is the top half of an fp32 pattern */
  return (double)f;
}

float oref_f64_to_f32(double x) { return (float)x; }

/* Array forms (for exhaustive checks). */
void oref_f64_to_f16_n(const double *x, int64_t n, uint16_t *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oref_f64_to_f16(x[i]);
}

void oref_f32_to_bf16_n(const float *x, int64_t n, uint16_t *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oref_f32_to_bf16(x[i]);
}

void oref_f16_to_f64_n(const uint16_t *h, int64_t n, double *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oref_f16_to_f64(h[i]);
}
