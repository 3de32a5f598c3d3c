/*
 * tq.h — packed ternary weight matmul for NVIDIA B200 (sm_100a): C ABI.
 *
 * Two weight formats:
 *
 *   TQ_FMT_A  group ternary ("Does your weight format deserve a kernel?",
 *             precisit.com). A group of G consecutive weights of a row shares
 *             an fp16 scale s = fp16(mean |W_j|) (section "Three values and a
 *             shared scale"); each weight is a trit t_j = clip(round(W_j/s),
 *             -1, 1), nearest-even ties, t = 0 for the whole group when s = 0.
 *             Five trits are packed per byte as b = d0 + 3 d1 + 9 d2 + 27 d3 +
 *             81 d4 with d = t + 1, first digit least significant (section
 *             "Five trits in a byte"); each group starts on a byte boundary, so
 *             a group takes ceil(G/5) code bytes (13 for G = 64) plus its 2-byte
 *             scale: 1.875 bits per weight at G = 64 (section "Count the bytes
 *             you actually wrote"). Padding digits hold 1 (trit 0). An optional
 *             second plane (FUCINA README, "The method": W ~ d1 T1 + d2 T2) is
 *             the same rule applied to the fp32 residual W - s1 t1.
 *             The decoded weight is w = s1 t1 [+ s2 t2].
 *
 *   TQ_FMT_B  ladder code book ("A Discrete Weight Language for Large Language
 *             Models", alphaneural.io). One uint8 code per weight (section 4.1)
 *             spells a word c in {-1,0,+1}^5, code = sum_i (c_i + 1) 3^(i-1)
 *             with c_1 least significant; the layer code book is
 *             LUT[code] = alpha * sum_i c_i a_i (section 3.2); an optional fp16
 *             scale rho per row or per block of rows multiplies the output
 *             accumulator (sections 3.3 and 4.2). The decoded weight is
 *             w = rho[n / rows_per_scale] * LUT[code] (rho = 1 when absent).
 *
 * Layouts (all row-major, C order):
 *   W      bf16 [n][k], contiguous.
 *   A      codes  uint8  [planes][n][k/G][ceil(G/5)]  (plane p starts at
 *                 codes + p * codes_plane_stride bytes; 0 = n*(k/G)*ceil(G/5))
 *          scales fp16   [planes][n][k/G]  (plane p at scales +
 *                 p * scales_plane_stride elements; 0 = n*(k/G))
 *   B      codes  uint8  [n][k];  lut fp32 [256] (entries 243..255 NaN);
 *          rho    fp16   [ceil(n / rows_per_scale)] or NULL
 *   B7     codes  uint8  [n][14 k / 16]: 7-bit indices, 16 per 14 bytes,
 *                 little-endian (index j of a chunk at bits 7j .. 7j + 6);
 *          lut    fp32   [128]: LUT7[i] = LUT[used[i]] (tq_build_lut7);
 *          rho as B (alphaneural.io page, section 8.1, the 7-bit truncated
 *          alphabet: a layer that uses at most 128 of the 243 words)
 *   x      bf16 [batch][ldx];  y fp32 [batch][ldy];  y = x * W_hat^T.
 *
 * Conventions:
 *   - Every buffer is allocated and owned by the caller. Pointers marked
 *     "device" must be device (or managed) memory of the current device.
 *   - GPU entry points enqueue work on `cuda_stream` (a cudaStream_t, NULL =
 *     legacy default stream) and return without synchronising. Their return
 *     value reports argument, shape and alignment errors (checked before any
 *     launch) and launch failures (TQ_ERR_CUDA).
 *   - Data errors found by a kernel (invalid code bytes, non-finite weights,
 *     fp16 scale overflow) are written to the optional device word
 *     `dev_status`: the first error code wins (atomic compare-and-swap from
 *     TQ_OK). The caller sets *dev_status = TQ_OK before the call and reads it
 *     after synchronising. With dev_status == NULL data errors go unreported.
 *   - The library keeps no device allocations. Its host state is a few
 *     per-process caches, each written once under std::call_once or an
 *     atomic (the driver's tensor-map encoder, a kernel's shared-memory limit
 *     per device, resident-cluster counts per device), and the test hooks of
 *     tq_testing.h. All entry points are reentrant and thread-safe.
 *   - Every wait inside a kernel is bounded (2 s). A wait that gives up ends
 *     the kernel's work early; tq_linear then leaves NaN in every output it
 *     could not finish, which is how a time-out is reported. TQ_ERR_TIMEOUT is
 *     reserved: no entry point returns it.
 *   - tq_linear's kernels are launched with programmatic dependent launch:
 *     one may begin its set-up (and hint the L2 cache with its first code
 *     bytes) while the kernel before it on the stream finishes, but it reads
 *     no user memory and writes nothing before that kernel has completed, so
 *     stream order holds as for any launch.
 *   - tq_linear is deterministic: for the same inputs, shapes and device,
 *     every output is bit-identical from call to call (partial sums are added
 *     in a fixed order).
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARG = 1, /* null pointer, bad count, bad enum value */
  TQ_ERR_SHAPE = 2,       /* k not a multiple of G / of 16, ld too small */
  TQ_ERR_ALIGNMENT = 3,   /* a pointer or stride breaks the alignment rule */
  TQ_ERR_UNSUPPORTED = 4, /* valid but unsupported parameter (e.g. G) */
  TQ_ERR_BAD_CODE = 5,    /* code byte >= 243, or a padding digit != 1 */
  TQ_ERR_NONFINITE = 6,   /* NaN or Inf in W */
  TQ_ERR_RANGE = 7,       /* a group mean rounds to fp16 infinity (>= 65520) */
  TQ_ERR_TIMEOUT = 8,     /* a bounded in-kernel wait gave up */
  TQ_ERR_CUDA = 9         /* a CUDA launch or runtime call failed */
} tq_status;

typedef enum {
  TQ_FMT_A = 1, /* group ternary, 5 trits per byte, fp16 group scales */
  TQ_FMT_B = 2, /* 243-entry ladder code book, one code per byte */
  TQ_FMT_B7 = 3 /* Format B over a used-code table: 7-bit indices */
} tq_format;

typedef struct {
  int32_t format;          /* tq_format */
  int32_t group;           /* A: G, 64 or 128, G divides k_cols. B: ignored */
  int32_t planes;          /* A: 1 or 2. B: must be 1 */
  int32_t rows_per_scale;  /* B: 0 = no rho; r > 0: row n uses rho[n / r] */
  int64_t n_rows;          /* N: rows of W (outputs) */
  int64_t k_cols;          /* K: columns of W (inputs). B: multiple of 16 */
  const uint8_t *codes;    /* device, 16-byte aligned; layout above */
  const uint16_t *scales;  /* device. A: fp16 group scales (required),
                              16-byte aligned. B: rho (fp16, 2-byte
                              aligned) or NULL */
  const float *lut;        /* B: device, 256 fp32 (tq_build_lut), 16-byte
                              aligned. B7: device, 128 fp32 (tq_build_lut7),
                              16-byte aligned. A: ignored */
  int64_t codes_plane_stride;  /* A: bytes between planes; 0 = dense */
  int64_t scales_plane_stride; /* A: elements between planes; 0 = dense */
  int64_t lut_rows;        /* B: 0 = one code book for every row; r > 0 =
                              adaptive alphabet (alphaneural.io page,
                              section 8.3): row n decodes with the code book
                              lut + 256 * (n / r), lut holding ceil(n / r)
                              books of 256 fp32 (one tq_build_lut per
                              block's ladder). A: must be 0 */
} tq_weights;

/* Bytes of a package: A = planes * n * (k/G) * (ceil(G/5) + 2) (codes and
 * scales; "Count the bytes you actually wrote"), B = n * k + 972 (codes and
 * the 243-entry table; rho excluded). Returns 0 for invalid arguments.
 * Host only; no GPU needed. */
size_t tq_packed_bytes(int32_t format, int64_t n, int64_t k, int32_t group,
                       int32_t planes);

/* Build the Format B layer code book on the host (alphaneural.io page,
 * section 3.2): lut_out[b] = fp32(alpha * S_b), S_b = sum_{i=1..5} c_i(b) a_i
 * accumulated in fp64 over ascending i, c_i(b) = ((b / 3^(i-1)) % 3) - 1,
 * a_i = ladder[i-1]; lut_out[243..255] = NaN. Host pointers; no GPU needed.
 * Errors: TQ_ERR_INVALID_ARG for NULL pointers. */
tq_status tq_build_lut(float alpha, const float ladder[5], float lut_out[256]);

/* Format A quantize and pack (precisit.com page, sections "Three values and a
 * shared scale" and "Five trits in a byte"; second plane per the FUCINA README,
 * "The method").
 *   W_bf16      device, bf16 [n][k] contiguous, 16-byte aligned.
 *   group       G = 64 or 128 (TQ_ERR_UNSUPPORTED otherwise); k % G == 0.
 *   planes      1 or 2. Plane 2 quantizes R = fp32(W - s1 t1) with the same G.
 *   codes_out   device, planes * n * (k/G) * ceil(G/5) bytes, dense planar
 *               layout, 16-byte aligned.
 *   scales_out  device, planes * n * (k/G) fp16, 4-byte aligned (tq_linear
 *               takes Format A scales 16-byte aligned: allocate for that).
 *   dev_status  device int32 or NULL: TQ_ERR_NONFINITE / TQ_ERR_RANGE.
 * Each group: S = sum |W_j| in fp64 over ascending j, s = fp16_RNE(S / G),
 * t_j = 0 if s == 0 else sign(W_j) [|W_j| > s/2]. Deterministic. */
tq_status tq_quantize_pack(const void *W_bf16, int64_t n, int64_t k,
                           int32_t group, int32_t planes, uint8_t *codes_out,
                           uint16_t *scales_out, int32_t *dev_status,
                           void *cuda_stream);

/* Format B encoder ("A Discrete Weight Language for Large Language Models",
 * alphaneural.io, section 3.1 "Encoding" and section 3.3 "Per-row scale").
 * Every weight x of W becomes the word c_1..c_5 of the greedy 5-step ternary
 * path over the ladder s_1..s_5 = ladder[0..4] of r_0 = x / a: step i keeps
 * c_i = 0 while |r_{i-1}| < zeta s_i (the zero bias), else takes the sign of
 * r_{i-1} when that moves r strictly closer to 0 (ties give 0); r_i =
 * r_{i-1} - c_i s_i; code = sum (c_i + 1) 3^(i-1). Decisions are made in
 * IEEE fp32: r_0 = fp32(x / a), threshold fp32(zeta s_i), r = fp32(r - c s).
 *   W_bf16          device, bf16 [n][k] contiguous, 16-byte aligned;
 *                   k % 16 == 0.
 *   ladder          host, 5 finite amplitudes > 0.
 *   zeta            zero bias in [0, 1]; 0.5 (or less) is the plain nearest
 *                   choice.
 *   rows_per_scale  0: a = alpha = max |W| over the matrix, no rho.
 *                   r > 0: a = max |W| over rows [g r, g r + r) of group
 *                   g = n / r (1: per row; the head size: per head) and
 *                   rho_out[g] = fp16(a / alpha) (0 for an all-zero group).
 *   codes_out       device, uint8 [n][k], 16-byte aligned.
 *   rho_out         device, fp16 [ceil(n / r)], 2-byte aligned (r > 0).
 *   alpha_out       device fp32: alpha = max |W| (build the code book with
 *                   tq_build_lut(alpha, ladder)).
 *   dev_status      device int32 or NULL: TQ_ERR_NONFINITE for NaN / Inf in
 *                   W (those weights are skipped by the maxima; their codes
 *                   are unspecified).
 * An all-zero group (or matrix) gives code 121 (the all-zero word).
 * Deterministic. */
tq_status tq_encode_b(const void *W_bf16, int64_t n, int64_t k,
                      const float ladder[5], float zeta,
                      int32_t rows_per_scale, uint8_t *codes_out,
                      uint16_t *rho_out, float *alpha_out, int32_t *dev_status,
                      void *cuda_stream);

/* Decode a package to bf16 (precisit.com page, "Three values and a shared
 * scale": W_hat = bf16(s t); alphaneural.io page, section 3.3).
 *   A: W_hat = bf16_RNE(fp32_RN(s1 t1 [+ s2 t2])).
 *   B: W_hat = bf16_RNE(fp32_RN(rho * LUT[code])), or bf16_RNE(LUT[code]).
 *   W_bf16_out  device, bf16 [n][k] contiguous, 16-byte aligned.
 *   dev_status  device int32 or NULL: TQ_ERR_BAD_CODE for a byte >= 243 or a
 *               Format A padding digit != 1 (the value written there is
 *               unspecified). */
tq_status tq_unpack(const tq_weights *w, void *W_bf16_out, int32_t *dev_status,
                    void *cuda_stream);

/* Fused packed matmul y = x * W_hat^T, decoding the codes inside the kernel
 * (precisit.com page, "What survives the round trip?": decode small pieces
 * inside a matrix multiplication; alphaneural.io page, section 4.2).
 *   A: y[b][n] = sum_p sum_g s_p[n][g] sum_{j in g} t_p[n][j] x[b][j]
 *   B: y[b][n] = rho[n / rows_per_scale] * sum_k LUT[code[n][k]] x[b][k]
 *   x     device, bf16 [batch][ldx], 16-byte aligned, ldx >= k, ldx % 8 == 0.
 *   y     device, fp32 [batch][ldy], 4-byte aligned, ldy >= n.
 *         Overwritten. fp32 accumulation.
 *   batch >= 1 (1..64 per pass; larger batches run in passes of 64).
 * Codes are not validated here (tq_unpack does that): a Format B code >= 243
 * reads a NaN table entry; an invalid Format A byte gives an unspecified
 * finite value. Accuracy: |y - y_exact| <= 2e-3 * ||x_b||_2 * max_k |w[n][k]|
 * where y_exact uses the exact decoded weights.
 * Format A reads: a row's codes and scales are fetched in whole 16-byte
 * blocks, from the block holding the first byte to the block holding the
 * last. A 16-byte block never crosses a page, so these reads stay in mapped
 * memory without padding; the bytes beyond the package are ignored.
 * A bounded wait that gives up leaves NaN in the outputs it could not finish
 * (the return value is still TQ_OK; see the conventions above). */
tq_status tq_linear(const tq_weights *w, const void *x_bf16, int64_t batch,
                    int64_t ldx, float *y, int64_t ldy, void *cuda_stream);

/* Expert-indexed Format A weights (FUCINA README, "The method": hot experts
 * carry both ternary planes W ~ d1 T1 + d2 T2, cold experts one; the experts
 * are stored hot-first, so the second plane covers the prefix 0 .. n_hot - 1).
 * Every expert is an n_rows x k_cols Format A matrix with group G = 64.
 *   codes / scales    plane 1 of every expert: expert e at
 *                     codes + e * n * (k/64) * 13 bytes and
 *                     scales + e * n * (k/64) fp16 (the Format A layout of
 *                     one plane); device, 16-byte aligned.
 *   codes2 / scales2  plane 2 of experts 0 .. n_hot - 1, same layout and
 *                     strides; NULL when n_hot = 0. */
typedef struct {
  int32_t n_experts;       /* E >= 1 */
  int32_t n_hot;           /* 0 .. E: experts with a second plane */
  int32_t group;           /* G: must be 64 */
  int32_t reserved;        /* 0 */
  int64_t n_rows;          /* N of every expert */
  int64_t k_cols;          /* K of every expert, a multiple of 64 */
  const uint8_t *codes;
  const uint16_t *scales;
  const uint8_t *codes2;
  const uint16_t *scales2;
} tq_experts;

/* Expert-indexed packed matmul (the mixture-of-experts product of the FUCINA
 * README; a token routed to k experts appears once per expert):
 *   y[t][n] = sum_k w_{ids[t]}[n][k] x[t][k],  w_e = s1 t1 + s2 t2 for
 *   e < n_hot, s1 t1 otherwise, for t = 0 .. n_tokens - 1.
 *   ids       device int32 [n_tokens], 4-byte aligned.
 *   x         device bf16 [n_tokens][ldx], 16-byte aligned, ldx >= k,
 *             ldx % 8 == 0.
 *   y         device fp32 [n_tokens][ldy], 4-byte aligned, ldy >= n.
 *   n_tokens  0 .. 65535 (0: nothing to do).
 *   dev_status device int32 or NULL: TQ_ERR_INVALID_ARG when an id lies
 *             outside 0 .. E - 1; that token's row of y is then NaN.
 * Same accuracy bound as tq_linear. The ids stay on the device: one launch,
 * no host synchronisation. Expert-indexed calls have no counterpart of the
 * tensor-core path: each token is one batch-1 product. */
tq_status tq_linear_experts(const tq_experts *w, const int32_t *ids,
                            int64_t n_tokens, const void *x_bf16, int64_t ldx,
                            float *y, int64_t ldy, int32_t *dev_status,
                            void *cuda_stream);

/* 7-bit truncated alphabet (alphaneural.io page, section 8.1): turn Format B
 * codes [n][k] (k % 16 == 0) into the layer's table of used codes and 7-bit
 * indices into it.
 *   codes        device uint8 [n][k], 16-byte aligned.
 *   used_out     device uint8 [128], 16-byte aligned: the distinct codes in
 *                ascending order, padded with 121 (the all-zero word); it
 *                also holds the call's intermediate set of codes present.
 *   n_used_out   device int32: the number of distinct codes.
 *   packed_out   device uint8 [n][14 k / 16], 2-byte aligned.
 *   dev_status   device int32 or NULL: TQ_ERR_RANGE when more than 128
 *                codes are in use (the packed output is then unspecified).
 * Three launches; no memory beyond the outputs. */
tq_status tq_pack7(const uint8_t *codes, int64_t n, int64_t k,
                   uint8_t *used_out, int32_t *n_used_out, uint8_t *packed_out,
                   int32_t *dev_status, void *cuda_stream);

/* The code book of a 7-bit layer on the host: lut7_out[i] = lut[used[i]]
 * (128 entries; lut is the layer's 256-entry Format B book). Host pointers;
 * no GPU needed. Errors: TQ_ERR_INVALID_ARG for NULL pointers. */
tq_status tq_build_lut7(const float lut[256], const uint8_t used[128],
                        float lut7_out[128]);

/* Static description of a status value. */
const char *tq_status_string(tq_status status);

#ifdef __cplusplus
}
#endif
#endif /* TQ_H */
