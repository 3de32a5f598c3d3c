/*
 * Format A oracle: group ternary quantization, base-3 packing, unpacking and
 * the fp64 reference matmul (test infrastructure only; see oref.h).
 *
 * Follows "Does your weight format deserve a kernel?" (precisit.com):
 *   - "Three values and a shared scale": a group of G consecutive weights
 *     shares s = fp16(mean |W_j|); each weight becomes t_j = clip(round(W_j/s),
 *     -1, 1) with nearest-even ties; a zero scale gives an all-zero group
 *     without dividing; reconstruction is bf16(s t_j).
 *   - "Five trits in a byte": digits d = t + 1 in {0,1,2}, byte
 *     b = d0 + 3 d1 + 9 d2 + 27 d3 + 81 d4 with the first digit least
 *     significant; values 243..255 are invalid; padding decodes to zero.
 *   - "Count the bytes you actually wrote": each group starts on a byte
 *     boundary, ceil(G/5) code bytes plus a 2-byte fp16 scale.
 * and, for the optional second plane, "FUCINA" section "The method"
 * (W ~ d1 T1 + d2 T2, ternary planes with fp16 scales).
 *
 * Readings where the pages leave a step open (each stated where it is used):
 *   R1 groups are G consecutive k inside one row of the n x k matrix;
 *   R2 the mean is the fp64 sum of |W_j| in ascending j, divided by G, then
 *      rounded once to fp16 (RNE, subnormals kept);
 *   R3 "round" rounds the exact quotient W/s: |W/s| < 1/2 gives 0, exactly
 *      1/2 ties to even (0), above 1/2 gives +-1 after clipping;
 *   R4 s == 0 gives t = 0 for the whole group (also when the mean underflows);
 *   R5 a non-finite weight is OREF_ERR_NONFINITE; a mean that rounds to fp16
 *      infinity (>= 65520) is OREF_ERR_RANGE;
 *   R6 weight j = 5m + i of a group is digit i of byte m; padding digits hold 1;
 *   R7 the package is planar: codes [planes][n][k/G][ceil(G/5)], then scales
 *      [planes][n][k/G];
 *   R8 plane 2 is plane-1 quantization applied to R = fp32(W - s1 t1)
 *      (greedy residual), with the same G;
 *   R9 the matmul uses the exact weight s1 t1 [+ s2 t2].
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include "oref.h"

int32_t oref_bytes_per_group(int32_t G) { return (G + 4) / 5; }

uint64_t oref_packed_bytes(int32_t format, int64_t n, int64_t k, int32_t G,
                           int32_t planes) {
  if (n < 0 || k < 0) return 0;
  if (format == OREF_FMT_A) {
    if (G <= 0 || k % G != 0 || planes < 1 || planes > 2) return 0;
    uint64_t groups = (uint64_t)n * (uint64_t)(k / G);
    return (uint64_t)planes * groups *
           ((uint64_t)oref_bytes_per_group(G) + 2u);
  }
  if (format == OREF_FMT_B) {
    return (uint64_t)n * (uint64_t)k + 243u * 4u;
  }
  return 0;
}

/* ---- base-3 packing (R6) ---------------------------------------------- */

void oref_pack_trits(const int8_t *t, int32_t G, uint8_t *out) {
  const int32_t nb = oref_bytes_per_group(G);
  for (int32_t m = 0; m < nb; ++m) {
    int value = 0;
    int power = 1;
    for (int i = 0; i < 5; ++i) {
      int32_t j = 5 * m + i;
      int digit = (j < G) ? (t[j] + 1) : 1; /* padding digit 1 = trit 0 */
      value += digit * power;
      power *= 3;
    }
    out[m] = (uint8_t)value;
  }
}

int oref_unpack_trits(const uint8_t *in, int32_t G, int8_t *t) {
  const int32_t nb = oref_bytes_per_group(G);
  int status = OREF_OK;
  for (int32_t m = 0; m < nb; ++m) {
    int b = in[m];
    if (b >= 243) status = OREF_ERR_BAD_CODE;
    int power = 1;
    for (int i = 0; i < 5; ++i) {
      int digit = (b / power) % 3;
      int32_t j = 5 * m + i;
      if (j < G) {
        t[j] = (int8_t)(digit - 1);
      } else if (digit != 1) {
        status = OREF_ERR_BAD_CODE; /* padding must decode to zero */
      }
      power *= 3;
    }
  }
  return status;
}

/* ---- quantization (R1-R5, R8) ------------------------------------------ */

static void set_status(int *status, int code) {
  if (*status == OREF_OK) *status = code; /* first error wins */
}

/* Quantize one group of G values (given exactly as fp64) to a scale and
 * trits. Returns the fp16 scale bits. */
static uint16_t quantize_group(const double *v, int32_t G, int8_t *t,
                               int *status) {
  double sum = 0.0;
  for (int32_t j = 0; j < G; ++j) {
    if (!isfinite(v[j])) set_status(status, OREF_ERR_NONFINITE);
    sum += fabs(v[j]); /* R2: fp64, ascending j */
  }
  double mean = sum / (double)G;
  uint16_t s_bits = oref_f64_to_f16(mean);
  double s = oref_f16_to_f64(s_bits);
  if (isinf(s) && isfinite(mean)) set_status(status, OREF_ERR_RANGE);
  double half = s / 2.0; /* exact */
  for (int32_t j = 0; j < G; ++j) {
    int8_t tj = 0;
    if (s != 0.0) {          /* R4 */
      if (fabs(v[j]) > half) /* R3: exact comparison with s/2 */
        tj = (v[j] < 0.0) ? (int8_t)-1 : (int8_t)1;
    }
    t[j] = tj;
  }
  return s_bits;
}

int oref_quantize_pack_A(const uint16_t *W, int64_t n, int64_t k, int32_t G,
                         int32_t planes, uint8_t *codes, uint16_t *scales) {
  if (!W || !codes || !scales) return OREF_ERR_INVALID_ARG;
  if (G <= 0 || n < 0 || k < 0 || planes < 1 || planes > 2)
    return OREF_ERR_INVALID_ARG;
  if (k % G != 0) return OREF_ERR_SHAPE;
  const int32_t nb = oref_bytes_per_group(G);
  const int64_t gpr = k / G; /* groups per row */
  const int64_t plane_groups = n * gpr;
  int status = OREF_OK;
  double *v = (double *)malloc(sizeof(double) * (size_t)G);
  int8_t *t = (int8_t *)malloc((size_t)G);
  if (!v || !t) {
    free(v);
    free(t);
    return OREF_ERR_INVALID_ARG;
  }
  for (int64_t r = 0; r < n; ++r) {
    for (int64_t g = 0; g < gpr; ++g) {
      const int64_t gi = r * gpr + g;
      const uint16_t *src = W + r * k + g * G;
      for (int32_t j = 0; j < G; ++j) v[j] = oref_bf16_to_f64(src[j]);
      for (int32_t p = 0; p < planes; ++p) {
        uint16_t s_bits = quantize_group(v, G, t, &status);
        scales[p * plane_groups + gi] = s_bits;
        oref_pack_trits(t, G, codes + (p * plane_groups + gi) * nb);
        if (p + 1 < planes) {
          /* R8: residual rounded to fp32. The difference of two fp32 values
           * computed in fp64 and then rounded to fp32 is the correctly
           * rounded fp32 difference (53 >= 2*24 + 2). */
          double s = oref_f16_to_f64(s_bits);
          for (int32_t j = 0; j < G; ++j)
            v[j] = (double)oref_f64_to_f32(v[j] - s * (double)t[j]);
        }
      }
    }
  }
  free(v);
  free(t);
  return status;
}

/* ---- decoding ------------------------------------------------------------ */

/* Decode row r of every plane into exact fp64 weights w[k]. */
static int decode_row_A(const uint8_t *codes, const uint16_t *scales,
                        int64_t n, int64_t k, int32_t G, int32_t planes,
                        int64_t r, double *w, int8_t *t) {
  const int32_t nb = oref_bytes_per_group(G);
  const int64_t gpr = k / G;
  const int64_t plane_groups = n * gpr;
  int status = OREF_OK;
  for (int64_t j = 0; j < k; ++j) w[j] = 0.0;
  for (int32_t p = 0; p < planes; ++p) {
    for (int64_t g = 0; g < gpr; ++g) {
      const int64_t gi = p * plane_groups + r * gpr + g;
      int st = oref_unpack_trits(codes + gi * nb, G, t);
      if (st != OREF_OK) set_status(&status, st);
      double s = oref_f16_to_f64(scales[gi]);
      for (int32_t j = 0; j < G; ++j) {
        /* R9: s1 t1 + s2 t2 is exact in fp64 (two fp16 magnitudes). */
        w[g * G + j] += (t[j] == 0) ? 0.0 : s * (double)t[j];
      }
    }
  }
  return status;
}

static int check_A(const uint8_t *codes, const uint16_t *scales, int64_t n,
                   int64_t k, int32_t G, int32_t planes) {
  if (!codes || !scales) return OREF_ERR_INVALID_ARG;
  if (G <= 0 || n < 0 || k < 0 || planes < 1 || planes > 2)
    return OREF_ERR_INVALID_ARG;
  if (k % G != 0) return OREF_ERR_SHAPE;
  return OREF_OK;
}

int oref_unpack_A(const uint8_t *codes, const uint16_t *scales, int64_t n,
                  int64_t k, int32_t G, int32_t planes, uint16_t *W_out) {
  int st = check_A(codes, scales, n, k, G, planes);
  if (st != OREF_OK) return st;
  if (!W_out) return OREF_ERR_INVALID_ARG;
  double *w = (double *)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
  int8_t *t = (int8_t *)malloc((size_t)G);
  int status = OREF_OK;
  for (int64_t r = 0; r < n; ++r) {
    int s = decode_row_A(codes, scales, n, k, G, planes, r, w, t);
    if (s != OREF_OK) set_status(&status, s);
    for (int64_t j = 0; j < k; ++j) {
      /* bf16(fp32(s1 t1 + s2 t2)): the exact sum rounded to fp32, then to
       * bf16 (two roundings, as the reconstruction is defined). */
      float f = oref_f64_to_f32(w[j]);
      W_out[r * k + j] = oref_f32_to_bf16(f);
    }
  }
  free(w);
  free(t);
  return status;
}

int oref_weights_A(const uint8_t *codes, const uint16_t *scales, int64_t n,
                   int64_t k, int32_t G, int32_t planes, const int64_t *rows,
                   int64_t nrows, double *w_out) {
  int st = check_A(codes, scales, n, k, G, planes);
  if (st != OREF_OK) return st;
  if (!w_out) return OREF_ERR_INVALID_ARG;
  if (!rows) nrows = n;
  int8_t *t = (int8_t *)malloc((size_t)G);
  int status = OREF_OK;
  for (int64_t i = 0; i < nrows; ++i) {
    int64_t r = rows ? rows[i] : i;
    if (r < 0 || r >= n) {
      free(t);
      return OREF_ERR_INVALID_ARG;
    }
    int s = decode_row_A(codes, scales, n, k, G, planes, r, w_out + i * k, t);
    if (s != OREF_OK) set_status(&status, s);
  }
  free(t);
  return status;
}

int oref_linear_A(const uint8_t *codes, const uint16_t *scales, int64_t n,
                  int64_t k, int32_t G, int32_t planes, const int64_t *rows,
                  int64_t nrows, const uint16_t *x, int64_t batch, int64_t ldx,
                  double *y) {
  int st = check_A(codes, scales, n, k, G, planes);
  if (st != OREF_OK) return st;
  if (!x || !y || batch < 0 || ldx < k) return OREF_ERR_INVALID_ARG;
  if (!rows) nrows = n;
  double *w = (double *)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
  int8_t *t = (int8_t *)malloc((size_t)G);
  int status = OREF_OK;
  for (int64_t i = 0; i < nrows; ++i) {
    int64_t r = rows ? rows[i] : i;
    if (r < 0 || r >= n) {
      status = OREF_ERR_INVALID_ARG;
      break;
    }
    int s = decode_row_A(codes, scales, n, k, G, planes, r, w, t);
    if (s != OREF_OK) set_status(&status, s);
    for (int64_t b = 0; b < batch; ++b) {
      const uint16_t *xb = x + b * ldx;
      double acc = 0.0;
      for (int64_t j = 0; j < k; ++j) acc += w[j] * oref_bf16_to_f64(xb[j]);
      y[b * nrows + i] = acc;
    }
  }
  free(w);
  free(t);
  return status;
}

/* ---- expert-indexed matmul (FUCINA README, "The method") -----------------
 *
 * A mixture-of-experts layer stores one Format A matrix per expert. Hot
 * experts carry both ternary planes, W ~ d1 T1 + d2 T2; cold experts carry
 * one. Experts are written hot-first, so the second plane covers the expert
 * prefix 0 .. n_hot - 1. Every token t is routed to one expert ids[t] (a
 * token routed to several experts appears once per expert) and
 *   y[t][n] = sum_k w_{ids[t]}[n][k] x[t][k],
 *   w_e = s1 t1 + s2 t2 (e < n_hot) or s1 t1 (e >= n_hot),
 * fp64, k ascending (the exact decoded weights, as oref_linear_A).
 * Layouts: plane 1 of expert e: codes1 + e * n * (k/G) * ceil(G/5) bytes,
 * scales1 + e * n * (k/G); plane 2 of expert e < n_hot: the same offsets in
 * codes2 / scales2. ids outside 0 .. n_experts - 1 are OREF_ERR_INVALID_ARG.
 * y: [n_tokens][n]. */
int oref_linear_experts_A(const uint8_t *codes1, const uint16_t *scales1,
                          const uint8_t *codes2, const uint16_t *scales2,
                          int32_t n_experts, int32_t n_hot, int64_t n,
                          int64_t k, int32_t G, const int32_t *ids,
                          int64_t n_tokens, const uint16_t *x, int64_t ldx,
                          double *y) {
  if (!codes1 || !scales1 || !ids || !x || !y) return OREF_ERR_INVALID_ARG;
  if (n_experts < 1 || n_hot < 0 || n_hot > n_experts || n_tokens < 0)
    return OREF_ERR_INVALID_ARG;
  if (n_hot > 0 && (!codes2 || !scales2)) return OREF_ERR_INVALID_ARG;
  if (ldx < k) return OREF_ERR_INVALID_ARG;
  const int st = check_A(codes1, scales1, n, k, G, 1);
  if (st != OREF_OK) return st;
  const int64_t gpr = k / G;
  const int64_t cstride = n * gpr * oref_bytes_per_group(G); /* bytes */
  const int64_t sstride = n * gpr;                           /* scales */
  double *w1 = (double *)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
  double *w2 = (double *)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
  int status = OREF_OK;
  for (int64_t t = 0; t < n_tokens; ++t) {
    const int32_t e = ids[t];
    if (e < 0 || e >= n_experts) {
      status = OREF_ERR_INVALID_ARG;
      break;
    }
    for (int64_t r = 0; r < n; ++r) {
      int s = oref_weights_A(codes1 + e * cstride, scales1 + e * sstride, n, k,
                             G, 1, &r, 1, w1);
      if (s != OREF_OK) set_status(&status, s);
      if (e < n_hot) {
        s = oref_weights_A(codes2 + e * cstride, scales2 + e * sstride, n, k,
                           G, 1, &r, 1, w2);
        if (s != OREF_OK) set_status(&status, s);
      }
      double acc = 0.0;
      for (int64_t j = 0; j < k; ++j) {
        /* s1 t1 + s2 t2: both terms are fp16 values times a trit; their
         * fp64 sum is exact */
        const double wj = e < n_hot ? w1[j] + w2[j] : w1[j];
        acc += wj * oref_bf16_to_f64(x[t * ldx + j]);
      }
      y[t * n + r] = acc;
    }
  }
  free(w1);
  free(w2);
  return status;
}
