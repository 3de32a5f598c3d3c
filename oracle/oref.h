/*
 * oref — plain, slow CPU oracle for packed ternary weights.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may include, link or
 * call this code: only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it. It shares no source with the CUDA library.
 *
 * Everything here is written to be read against the pages it follows:
 *   - "Does your weight format deserve a kernel?" (precisit.com), sections
 *     "Three values and a shared scale" (the scale rule s = fp16(mean|W|) and
 *     the trit rule t = clip(round(W/s), -1, 1) with nearest-even ties) and
 *     "Five trits in a byte" (b = d0 + 3 d1 + 9 d2 + 27 d3 + 81 d4, first digit
 *     least significant; bytes 243..255 rejected; padding decodes to zero) and
 *     "Count the bytes you actually wrote" (byte-aligned groups, 13 code bytes
 *     plus an fp16 scale per 64 weights).
 *   - "A Discrete Weight Language for Large Language Models" (alphaneural.io),
 *     section 3.2 (the 243-entry layer code book LUT = alpha * sum c_i s_i),
 *     section 3.3 (per-row scale rho, W_hat = rho * LUT[code]) and section 4.2
 *     (rho applied to the output accumulator).
 *   - "FUCINA" (git mirror README), section "The method" (W ~ d1 T1 + d2 T2,
 *     two ternary planes with fp16 scales).
 *
 * Floating point: all arithmetic is IEEE fp64 unless a step names another
 * precision. fp16 and bf16 rounding are implemented here from the IEEE-754
 * definition (round to nearest, ties to even, subnormals kept), not taken from
 * a library. Build with -ffp-contract=off and without -ffast-math.
 *
 * Status values returned by these functions (0 = success) use the same
 * numbering as the library's status enum, but are defined independently.
 */
#ifndef OREF_H
#define OREF_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  OREF_OK = 0,
  OREF_ERR_INVALID_ARG = 1,
  OREF_ERR_SHAPE = 2,
  OREF_ERR_UNSUPPORTED = 4,
  OREF_ERR_BAD_CODE = 5,
  OREF_ERR_NONFINITE = 6,
  OREF_ERR_RANGE = 7
};

enum { OREF_FMT_A = 1, OREF_FMT_B = 2 };

/* ---- IEEE binary16 / bfloat16 rounding (oref_fp.c) ---------------------- */
uint16_t oref_f64_to_f16(double x);   /* RNE, subnormals, overflow -> inf */
double oref_f16_to_f64(uint16_t h);   /* exact */
uint16_t oref_f64_to_bf16(double x);  /* RNE, subnormals, overflow -> inf */
uint16_t oref_f32_to_bf16(float x);   /* RNE; x is exact in fp64 */
double oref_bf16_to_f64(uint16_t b);  /* exact */
float oref_f64_to_f32(double x);      /* host IEEE conversion (RNE) */
void oref_f64_to_f16_n(const double *x, int64_t n, uint16_t *out);
void oref_f32_to_bf16_n(const float *x, int64_t n, uint16_t *out);
void oref_f16_to_f64_n(const uint16_t *h, int64_t n, double *out);

/* ---- Format A: group ternary, 5 trits per byte (oref_format_a.c) -------- */
int32_t oref_bytes_per_group(int32_t G);  /* ceil(G / 5) */
/* Total package bytes (codes + fp16 scales) for format A, or codes + LUT
 * (972 B) for format B (rho excluded: it depends on rows_per_scale). */
uint64_t oref_packed_bytes(int32_t format, int64_t n, int64_t k, int32_t G,
                           int32_t planes);

/* Pack one group of G trits (values -1, 0, +1) into ceil(G/5) bytes. */
void oref_pack_trits(const int8_t *t, int32_t G, uint8_t *out);
/* Unpack one group; returns OREF_ERR_BAD_CODE for a byte >= 243 or a padding
 * digit that is not 1 (trit 0). Trits are written even on error. */
int oref_unpack_trits(const uint8_t *in, int32_t G, int8_t *t);

/* Quantize and pack W (bf16 bits, [n][k] row-major) into
 *   codes  [planes][n][k/G][ceil(G/5)]  and  scales [planes][n][k/G] (fp16).
 * planes = 2 fits the second plane to the fp32 residual of the first. */
int oref_quantize_pack_A(const uint16_t *W, int64_t n, int64_t k, int32_t G,
                         int32_t planes, uint8_t *codes, uint16_t *scales);

/* Decode the package to bf16 W_hat = bf16(fp32(s1 t1 [+ s2 t2])). */
int oref_unpack_A(const uint8_t *codes, const uint16_t *scales, int64_t n,
                  int64_t k, int32_t G, int32_t planes, uint16_t *W_out);

/* Exact decoded weights w = s1 t1 [+ s2 t2] (fp64) of the listed rows
 * (rows == NULL: all rows, nrows ignored). Output [nrows][k]. */
int oref_weights_A(const uint8_t *codes, const uint16_t *scales, int64_t n,
                   int64_t k, int32_t G, int32_t planes, const int64_t *rows,
                   int64_t nrows, double *w_out);

/* y[b][i] = sum_k w[rows[i]][k] * x[b][k], fp64, k ascending.
 * x: bf16 bits, [batch][ldx]. y: fp64, [batch][nrows] dense. */
int oref_linear_A(const uint8_t *codes, const uint16_t *scales, int64_t n,
                  int64_t k, int32_t G, int32_t planes, const int64_t *rows,
                  int64_t nrows, const uint16_t *x, int64_t batch, int64_t ldx,
                  double *y);

/* Expert-indexed matmul (FUCINA README, "The method"): one Format A matrix
 * per expert, the second plane only on the hot-expert prefix 0..n_hot-1;
 * token t uses expert ids[t]: y[t][n] = sum_k w_{ids[t]}[n][k] x[t][k] (fp64,
 * exact decoded weights). Plane p of expert e at codes_p + e * n * (k/G) *
 * ceil(G/5) and scales_p + e * n * (k/G). y: [n_tokens][n]. */
int oref_linear_experts_A(const uint8_t *codes1, const uint16_t *scales1,
                          const uint8_t *codes2, const uint16_t *scales2,
                          int32_t n_experts, int32_t n_hot, int64_t n,
                          int64_t k, int32_t G, const int32_t *ids,
                          int64_t n_tokens, const uint16_t *x, int64_t ldx,
                          double *y);

/* ---- Format B: 243-entry ladder code book, one code per byte ------------ */
/* LUT[b] = fp32(alpha * sum_{i=1..5} c_i(b) a_i), sum in fp64 over i
 * ascending, c_i(b) = (i-1)-th base-3 digit of b minus 1 (first digit least
 * significant). lut[243..255] = NaN. */
int oref_build_lut(float alpha, const float ladder[5], float lut[256]);

/* W_hat = bf16(fp32(rho[n / rps] * LUT[code])) (rps > 0) or bf16(LUT[code]). */
int oref_unpack_B(const uint8_t *codes, int64_t n, int64_t k, const float *lut,
                  const uint16_t *rho, int32_t rps, uint16_t *W_out);

int oref_weights_B(const uint8_t *codes, int64_t n, int64_t k, const float *lut,
                   const uint16_t *rho, int32_t rps, const int64_t *rows,
                   int64_t nrows, double *w_out);

int oref_linear_B(const uint8_t *codes, int64_t n, int64_t k, const float *lut,
                  const uint16_t *rho, int32_t rps, const int64_t *rows,
                  int64_t nrows, const uint16_t *x, int64_t batch, int64_t ldx,
                  double *y);

/* Adaptive alphabets (section 8.3): the same with one code book per block of
 * lut_rows rows (row n uses lut + 256 * (n / lut_rows)); lut_rows = 0 is the
 * layer's single code book (the functions above). */
int oref_unpack_Bx(const uint8_t *codes, int64_t n, int64_t k,
                   const float *lut, int64_t lut_rows, const uint16_t *rho,
                   int32_t rps, uint16_t *W_out);
int oref_weights_Bx(const uint8_t *codes, int64_t n, int64_t k,
                    const float *lut, int64_t lut_rows, const uint16_t *rho,
                    int32_t rps, const int64_t *rows, int64_t nrows,
                    double *w_out);
int oref_linear_Bx(const uint8_t *codes, int64_t n, int64_t k,
                   const float *lut, int64_t lut_rows, const uint16_t *rho,
                   int32_t rps, const int64_t *rows, int64_t nrows,
                   const uint16_t *x, int64_t batch, int64_t ldx, double *y);

/* 7-bit truncated alphabet (section 8.1): `used` = the distinct codes in
 * ascending order (<= 128, else OREF_ERR_RANGE; padded with 121), 16 indices
 * into it per 14 bytes, little-endian (index j at bits 7j .. 7j+6), rows of
 * 14 k / 16 bytes (k % 16 == 0). unpack7_codes inverts pack7 to codes. */
int oref_pack7(const uint8_t *codes, int64_t n, int64_t k, uint8_t used[128],
               int32_t *n_used, uint8_t *packed);
int oref_unpack7_codes(const uint8_t *packed, const uint8_t used[128],
                       int64_t n, int64_t k, uint8_t *codes);

/* Encoder (section 3.1; per-row / per-head scale, section 3.3): the greedy
 * 5-step ternary path of every weight over the ladder with zero-bias zeta,
 * r_0 = W / a with a = alpha = max |W| (rps = 0) or a = max |W| over the
 * rows n / rps (rps > 0, then rho[g] = fp16(a_g / alpha)). Decisions in fp32.
 * codes [n][k]; rho [ceil(n / rps)] (rps > 0); *alpha_out = alpha. */
int oref_encode_B(const uint16_t *W, int64_t n, int64_t k,
                  const float ladder[5], float zeta, int32_t rps,
                  uint8_t *codes, uint16_t *rho, float *alpha_out);

#ifdef __cplusplus
}
#endif
#endif /* OREF_H */
