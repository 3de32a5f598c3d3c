/*
 * Format B oracle: the 243-word ternary code book, unpacking and the fp64
 * reference matmul (test infrastructure only; see oref.h).
 *
 * Follows "A Discrete Weight Language for Large Language Models"
 * (alphaneural.io):
 *   - section 3.2: a weight is the word c = (c_1..c_5) in {-1,0,+1}^5 and
 *     decodes to alpha * sum_i c_i s_i; the 243 words are enumerated once per
 *     layer, multiplied by alpha and stored as a 243-entry table; the weight
 *     matrix is then the matrix of codes in 0..242 (base-3 encoding of the
 *     word);
 *   - section 3.3: with a per-row scale rho_n (fp16), W_hat = rho_n LUT[code];
 *   - section 4.1: one uint8 code per weight (8 bits of storage);
 *   - section 4.2: rho is applied to the output accumulator.
 *
 * Readings where the page leaves a step open:
 *   B1 the digit order of the code is the one of the five-trits-per-byte
 *      layout: code = sum_i (c_i + 1) 3^(i-1), c_1 least significant;
 *   B2 the table is LUT[b] = fp32(alpha * S_b), S_b = sum_{i=1..5} c_i a_i in
 *      fp64 over ascending i, the ladder a_i and alpha given as fp32;
 *      entries 243..255 of the padded 256-entry table are NaN;
 *   B3 rho is optional; row n uses rho[n / rows_per_scale] (per row when
 *      rows_per_scale = 1, per attention head when it is the head size);
 *   B4 unpack yields bf16(fp32(rho * LUT[code])), or bf16(LUT[code]) without
 *      rho; codes >= 243 are OREF_ERR_BAD_CODE;
 *   B5 the matmul uses the exact weight rho * LUT[code] (fp64).
 *
 * Adaptive alphabets (section 8.3 "Adaptive alphabets": one ladder per row
 * or per block of 32 rows instead of one per layer), read as one code book
 * per block of lut_rows rows: row n decodes with the table
 * lut + 256 * (n / lut_rows), each built from its block's ladder as above;
 * lut_rows = 0 is the single code book of the layer.
 */
#include <math.h>
#include <stdlib.h>

#include "oref.h"

int oref_build_lut(float alpha, const float ladder[5], float lut[256]) {
  if (!ladder || !lut) return OREF_ERR_INVALID_ARG;
  for (int b = 0; b < 243; ++b) {
    double sum = 0.0;
    int rest = b;
    for (int i = 0; i < 5; ++i) { /* i = 0 is c_1, the least significant */
      int c = rest % 3 - 1;
      rest /= 3;
      sum += (double)c * (double)ladder[i];
    }
    lut[b] = oref_f64_to_f32((double)alpha * sum);
  }
  for (int b = 243; b < 256; ++b) lut[b] = NAN;
  return OREF_OK;
}

static int check_B(const uint8_t *codes, int64_t n, int64_t k,
                   const float *lut, int64_t lut_rows, const uint16_t *rho,
                   int32_t rps) {
  if (!codes || !lut || n < 0 || k < 0) return OREF_ERR_INVALID_ARG;
  if (rps < 0 || lut_rows < 0) return OREF_ERR_INVALID_ARG;
  if (rps > 0 && !rho) return OREF_ERR_INVALID_ARG;
  return OREF_OK;
}

/* the code book of row r */
static const float *row_lut(const float *lut, int64_t lut_rows, int64_t r) {
  return lut_rows > 0 ? lut + 256 * (r / lut_rows) : lut;
}

int oref_unpack_Bx(const uint8_t *codes, int64_t n, int64_t k,
                   const float *lut, int64_t lut_rows, const uint16_t *rho,
                   int32_t rps, uint16_t *W_out) {
  int st = check_B(codes, n, k, lut, lut_rows, rho, rps);
  if (st != OREF_OK) return st;
  if (!W_out) return OREF_ERR_INVALID_ARG;
  int status = OREF_OK;
  for (int64_t r = 0; r < n; ++r) {
    double scale = (rps > 0) ? oref_f16_to_f64(rho[r / rps]) : 1.0;
    const float *L = row_lut(lut, lut_rows, r);
    for (int64_t j = 0; j < k; ++j) {
      uint8_t c = codes[r * k + j];
      if (c >= 243 && status == OREF_OK) status = OREF_ERR_BAD_CODE;
      double v = (double)L[c];
      /* rho * LUT: fp16 x fp32 is exact in fp64, then rounded to fp32 */
      float f = (rps > 0) ? oref_f64_to_f32(scale * v) : (float)v;
      W_out[r * k + j] = oref_f32_to_bf16(f);
    }
  }
  return status;
}

int oref_unpack_B(const uint8_t *codes, int64_t n, int64_t k, const float *lut,
                  const uint16_t *rho, int32_t rps, uint16_t *W_out) {
  return oref_unpack_Bx(codes, n, k, lut, 0, rho, rps, W_out);
}

int oref_weights_Bx(const uint8_t *codes, int64_t n, int64_t k,
                    const float *lut, int64_t lut_rows, const uint16_t *rho,
                    int32_t rps, const int64_t *rows, int64_t nrows,
                    double *w_out) {
  int st = check_B(codes, n, k, lut, lut_rows, rho, rps);
  if (st != OREF_OK) return st;
  if (!w_out) return OREF_ERR_INVALID_ARG;
  if (!rows) nrows = n;
  int status = OREF_OK;
  for (int64_t i = 0; i < nrows; ++i) {
    int64_t r = rows ? rows[i] : i;
    if (r < 0 || r >= n) return OREF_ERR_INVALID_ARG;
    double scale = (rps > 0) ? oref_f16_to_f64(rho[r / rps]) : 1.0;
    const float *L = row_lut(lut, lut_rows, r);
    for (int64_t j = 0; j < k; ++j) {
      uint8_t c = codes[r * k + j];
      if (c >= 243 && status == OREF_OK) status = OREF_ERR_BAD_CODE;
      w_out[i * k + j] = scale * (double)L[c]; /* exact (B5) */
    }
  }
  return status;
}

int oref_weights_B(const uint8_t *codes, int64_t n, int64_t k, const float *lut,
                   const uint16_t *rho, int32_t rps, const int64_t *rows,
                   int64_t nrows, double *w_out) {
  return oref_weights_Bx(codes, n, k, lut, 0, rho, rps, rows, nrows, w_out);
}

int oref_linear_Bx(const uint8_t *codes, int64_t n, int64_t k,
                   const float *lut, int64_t lut_rows, const uint16_t *rho,
                   int32_t rps, const int64_t *rows, int64_t nrows,
                   const uint16_t *x, int64_t batch, int64_t ldx, double *y) {
  int st = check_B(codes, n, k, lut, lut_rows, rho, rps);
  if (st != OREF_OK) return st;
  if (!x || !y || batch < 0 || ldx < k) return OREF_ERR_INVALID_ARG;
  if (!rows) nrows = n;
  double *w = (double *)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
  int status = OREF_OK;
  for (int64_t i = 0; i < nrows; ++i) {
    int64_t r = rows ? rows[i] : i;
    if (r < 0 || r >= n) {
      status = OREF_ERR_INVALID_ARG;
      break;
    }
    int s = oref_weights_Bx(codes, n, k, lut, lut_rows, rho, rps, &r, 1, w);
    if (s != OREF_OK && status == OREF_OK) status = s;
    for (int64_t b = 0; b < batch; ++b) {
      const uint16_t *xb = x + b * ldx;
      double acc = 0.0;
      for (int64_t j = 0; j < k; ++j) acc += w[j] * oref_bf16_to_f64(xb[j]);
      y[b * nrows + i] = acc;
    }
  }
  free(w);
  return status;
}

int oref_linear_B(const uint8_t *codes, int64_t n, int64_t k, const float *lut,
                  const uint16_t *rho, int32_t rps, const int64_t *rows,
                  int64_t nrows, const uint16_t *x, int64_t batch, int64_t ldx,
                  double *y) {
  return oref_linear_Bx(codes, n, k, lut, 0, rho, rps, rows, nrows, x, batch,
                        ldx, y);
}

/* ---- encoder (section 3.1 "Encoding", section 3.3 "Per-row scale") -------
 *
 * The page's greedy 5-step ternary path: with the residual r_0 = x / a, step
 * i picks c_i in {-1, 0, +1} minimising |r_{i-1} - c s_i|, except that a
 * zero-bias zeta prefers c_i = 0 when |r_{i-1}| < zeta s_i, and leaves the
 * residual r_i = r_{i-1} - c_i s_i. The scale a is the global alpha =
 * max |W| (section 3.1), or, with a per-row (or per-head) scale, the maximum
 * |W| over the row (or the head's rows), alpha_n, with rho_n = alpha_n / alpha
 * stored in fp16 (section 3.3).
 *
 * Readings where the page leaves a step open:
 *   E1 precision: the page fixes none; every step that decides a digit runs
 *      in IEEE fp32 in the order written here: r_0 = fp32(x / a); the zero
 *      bias threshold is fp32(zeta * s_i); the non-zero candidate is the one
 *      with the sign of r (the nearer of -1 and +1), taken only when
 *      |fp32(r - c s_i)| < |r| strictly (a tie, and r = 0, give 0); then
 *      r = fp32(r - c_i s_i);
 *   E2 the scale group of row n is n / rows_per_scale (1: per row; the head
 *      size: per head), one alpha_g and one rho per group, as the rho layout
 *      of the matmul (B3); rows_per_scale = 0 uses the global alpha, no rho;
 *   E3 rho_g = fp16(alpha_g / alpha): the fp64 quotient rounded once to fp16;
 *   E4 a zero scale (an all-zero group, or an all-zero matrix) gives the
 *      all-zero word (code 121) and rho = 0;
 *   E5 alpha = max |W| is a bf16 magnitude, exact in fp32; NaN or Inf in W is
 *      OREF_ERR_NONFINITE (the outputs are then unspecified).
 */
static uint8_t encode_word(float r, const float s[5], const float zs[5]) {
  int code = 0, p3 = 1;
  for (int i = 0; i < 5; ++i) { /* step i + 1 of the path */
    int c = 0;
    const float ar = fabsf(r);
    if (!(ar < zs[i])) {
      const int cand = r > 0.0f ? 1 : (r < 0.0f ? -1 : 0);
      if (cand != 0) {
        const float rn = r - (float)cand * s[i];
        if (fabsf(rn) < ar) {
          c = cand;
          r = rn;
        }
      }
    }
    code += (c + 1) * p3; /* c_1 is the least significant digit (B1) */
    p3 *= 3;
  }
  return (uint8_t)code;
}

int oref_encode_B(const uint16_t *W, int64_t n, int64_t k,
                  const float ladder[5], float zeta, int32_t rps,
                  uint8_t *codes, uint16_t *rho, float *alpha_out) {
  if (!W || !ladder || !codes || !alpha_out || n < 0 || k < 0 || rps < 0)
    return OREF_ERR_INVALID_ARG;
  if (rps > 0 && !rho) return OREF_ERR_INVALID_ARG;
  int status = OREF_OK;
  /* alpha = max |W| over the whole matrix */
  double amax = 0.0;
  for (int64_t i = 0; i < n * k; ++i) {
    const double v = fabs(oref_bf16_to_f64(W[i]));
    if (!isfinite(v)) {
      status = OREF_ERR_NONFINITE;
      continue;
    }
    if (v > amax) amax = v;
  }
  const float alpha = (float)amax; /* exact (E5) */
  *alpha_out = alpha;
  float s[5], zs[5];
  for (int i = 0; i < 5; ++i) {
    s[i] = ladder[i];
    zs[i] = zeta * ladder[i]; /* fp32 product (E1) */
  }
  const int64_t group_rows = rps > 0 ? rps : (n > 0 ? n : 1);
  for (int64_t g0 = 0; g0 < n; g0 += group_rows) {
    const int64_t g1 = g0 + group_rows < n ? g0 + group_rows : n;
    float a = alpha;
    if (rps > 0) {
      double gmax = 0.0;
      for (int64_t i = g0 * k; i < g1 * k; ++i) {
        const double v = fabs(oref_bf16_to_f64(W[i]));
        if (isfinite(v) && v > gmax) gmax = v;
      }
      a = (float)gmax;
      rho[g0 / rps] = a == 0.0f ? 0 : oref_f64_to_f16((double)a / (double)alpha);
    }
    for (int64_t i = g0 * k; i < g1 * k; ++i) {
      const float x = (float)oref_bf16_to_f64(W[i]);
      const float r0 = a == 0.0f ? 0.0f : x / a; /* E1, E4 */
      codes[i] = encode_word(r0, s, zs);
    }
  }
  return status;
}

/* ---- 7-bit truncated alphabet (section 8.1 "Variable-depth words") --------
 *
 * When a layer uses only a few of the 243 words, a code fits in 7 bits
 * next to a per-layer table of the words in use. Readings where the page
 * leaves a step open:
 *   T1 the table `used` lists the distinct codes of the layer in ascending
 *      order, at most 128 of them (more is OREF_ERR_RANGE); entries past the
 *      count hold 121, the all-zero word;
 *   T2 a weight stores the index of its code in that table;
 *   T3 16 indices are packed little-endian into 14 bytes: index j of a
 *      chunk occupies bits 7j .. 7j + 6 of the chunk read as a 112-bit
 *      integer whose byte 0 holds bits 0 .. 7; a row of k codes (k a multiple
 *      of 16) takes 14 k / 16 bytes, rows back to back;
 *   T4 index i decodes to the code used[i], so the weight is LUT[used[i]]
 *      (times rho as in Format B) and the matmul is Format B's.
 */
int oref_pack7(const uint8_t *codes, int64_t n, int64_t k, uint8_t used[128],
               int32_t *n_used, uint8_t *packed) {
  if (!codes || !used || !n_used || !packed || n < 0 || k < 0 || k % 16 != 0)
    return OREF_ERR_INVALID_ARG;
  int present[256] = {0};
  for (int64_t i = 0; i < n * k; ++i) present[codes[i]] = 1;
  int count = 0;
  int index_of[256];
  for (int c = 0; c < 256; ++c) {
    index_of[c] = -1;
    if (present[c]) {
      if (count == 128) return OREF_ERR_RANGE;
      index_of[c] = count;
      used[count++] = (uint8_t)c;
    }
  }
  for (int i = count; i < 128; ++i) used[i] = 121;
  *n_used = count;
  const int64_t row_bytes = 14 * (k / 16);
  for (int64_t r = 0; r < n; ++r) {
    for (int64_t ch = 0; ch < k / 16; ++ch) {
      uint8_t *out = packed + r * row_bytes + 14 * ch;
      for (int b = 0; b < 14; ++b) out[b] = 0;
      for (int j = 0; j < 16; ++j) {
        const int idx = index_of[codes[r * k + 16 * ch + j]];
        for (int bit = 0; bit < 7; ++bit) /* bit 7j + bit of the chunk */
          if ((idx >> bit) & 1) {
            const int pos = 7 * j + bit;
            out[pos / 8] |= (uint8_t)(1u << (pos % 8));
          }
      }
    }
  }
  return OREF_OK;
}

int oref_unpack7_codes(const uint8_t *packed, const uint8_t used[128],
                       int64_t n, int64_t k, uint8_t *codes) {
  if (!packed || !used || !codes || n < 0 || k < 0 || k % 16 != 0)
    return OREF_ERR_INVALID_ARG;
  const int64_t row_bytes = 14 * (k / 16);
  for (int64_t r = 0; r < n; ++r) {
    for (int64_t ch = 0; ch < k / 16; ++ch) {
      const uint8_t *in = packed + r * row_bytes + 14 * ch;
      for (int j = 0; j < 16; ++j) {
        int idx = 0;
        for (int bit = 0; bit < 7; ++bit) {
          const int pos = 7 * j + bit;
          idx |= ((in[pos / 8] >> (pos % 8)) & 1) << bit;
        }
        codes[r * k + 16 * ch + j] = used[idx];
      }
    }
  }
  return OREF_OK;
}
