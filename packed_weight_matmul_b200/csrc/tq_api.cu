// C ABI of the tq library: argument validation, the host-side code book
// builder and dispatch to the kernels. Every check here happens before any
// launch; kernels report data errors through the caller's status word.
#include <math.h>
#include <string.h>

#include "tq_common.cuh"
#include "tq_linear.cuh"
#include "tq_testing.h"

namespace {

bool aligned(const void *p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

tq_status from_cuda(cudaError_t e) {
  return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

// Validate a weight descriptor; fills `v` on success.
tq_status check_weights(const tq_weights *w, tq::WeightsView *v) {
  if (w == nullptr) return TQ_ERR_INVALID_ARG;
  if (w->n_rows < 0 || w->k_cols < 0) return TQ_ERR_INVALID_ARG;
  if (w->codes == nullptr) return TQ_ERR_INVALID_ARG;
  v->format = w->format;
  v->n = w->n_rows;
  v->k = w->k_cols;
  v->codes = w->codes;
  v->scales = w->scales;
  v->lut = w->lut;
  v->group = w->group;
  v->planes = w->planes;
  v->rps = w->rows_per_scale;
  v->codes_plane_stride = 0;
  v->scales_plane_stride = 0;
  v->lut_rows = w->lut_rows;
  if (w->lut_rows < 0) return TQ_ERR_INVALID_ARG;
  if (w->format == TQ_FMT_A) {
    if (w->lut_rows != 0) return TQ_ERR_INVALID_ARG;
    if (w->scales == nullptr) return TQ_ERR_INVALID_ARG;
    if (w->planes < 1 || w->planes > 2) return TQ_ERR_INVALID_ARG;
    if (w->group != 64 && w->group != 128) return TQ_ERR_UNSUPPORTED;
    if (w->k_cols % w->group != 0) return TQ_ERR_SHAPE;
    const int64_t groups = w->n_rows * (w->k_cols / w->group);
    const int64_t nb = tq::bytes_per_group(w->group);
    v->codes_plane_stride =
        w->codes_plane_stride ? w->codes_plane_stride : groups * nb;
    v->scales_plane_stride =
        w->scales_plane_stride ? w->scales_plane_stride : groups;
    if (w->planes == 2 && (v->codes_plane_stride < groups * nb ||
                           v->scales_plane_stride < groups))
      return TQ_ERR_SHAPE;
    if (w->codes_plane_stride < 0 || w->scales_plane_stride < 0)
      return TQ_ERR_INVALID_ARG;
    // scales 16-byte aligned: kernels fetch them in aligned 16-byte chunks
    if (!aligned(w->codes, 16) || !aligned(w->scales, 16))
      return TQ_ERR_ALIGNMENT;
  } else if (w->format == TQ_FMT_B7) {
    // 7-bit indices into a used-code table, rows of 14 k / 16 bytes
    if (w->planes != 1 || w->lut_rows != 0) return TQ_ERR_INVALID_ARG;
    if (w->lut == nullptr) return TQ_ERR_INVALID_ARG;
    if (w->rows_per_scale < 0) return TQ_ERR_INVALID_ARG;
    if (w->rows_per_scale > 0 && w->scales == nullptr)
      return TQ_ERR_INVALID_ARG;
    if (w->k_cols % 16 != 0) return TQ_ERR_SHAPE;
    if (!aligned(w->codes, 2) || !aligned(w->lut, 16)) return TQ_ERR_ALIGNMENT;
    if (w->scales != nullptr && !aligned(w->scales, 2)) return TQ_ERR_ALIGNMENT;
    v->group = 0;
    if (w->rows_per_scale == 0) v->scales = nullptr;
  } else if (w->format == TQ_FMT_B) {
    if (w->planes != 1) return TQ_ERR_INVALID_ARG;
    if (w->lut == nullptr) return TQ_ERR_INVALID_ARG;
    if (w->rows_per_scale < 0) return TQ_ERR_INVALID_ARG;
    if (w->rows_per_scale > 0 && w->scales == nullptr)
      return TQ_ERR_INVALID_ARG;
    if (w->k_cols % 16 != 0) return TQ_ERR_SHAPE;
    if (!aligned(w->codes, 16) || !aligned(w->lut, 16)) return TQ_ERR_ALIGNMENT;
    if (w->scales != nullptr && !aligned(w->scales, 2)) return TQ_ERR_ALIGNMENT;
    v->group = 0;
    if (w->rows_per_scale == 0) v->scales = nullptr;
  } else {
    return TQ_ERR_INVALID_ARG;
  }
  return TQ_OK;
}

}  // namespace

extern "C" {

size_t tq_packed_bytes(int32_t format, int64_t n, int64_t k, int32_t group,
                       int32_t planes) {
  if (n < 0 || k < 0) return 0;
  if (format == TQ_FMT_A) {
    if (group <= 0 || k % group != 0 || planes < 1 || planes > 2) return 0;
    const size_t groups = (size_t)n * (size_t)(k / group);
    return (size_t)planes * groups * ((size_t)tq::bytes_per_group(group) + 2);
  }
  if (format == TQ_FMT_B) return (size_t)n * (size_t)k + 243u * 4u;
  if (format == TQ_FMT_B7) {
    if (k % 16 != 0) return 0;
    return (size_t)n * (size_t)(14 * (k / 16)) + 128u * 4u;
  }
  return 0;
}

tq_status tq_build_lut(float alpha, const float ladder[5], float lut_out[256]) {
  if (ladder == nullptr || lut_out == nullptr) return TQ_ERR_INVALID_ARG;
  for (int code = 0; code < 243; ++code) {
    // c_1 is the least significant base-3 digit of the code.
    double acc = 0.0;
    int digits = code;
    for (int i = 0; i < 5; ++i) {
      const int c = digits % 3 - 1;
      digits /= 3;
      acc += (double)c * (double)ladder[i];
    }
    lut_out[code] = (float)((double)alpha * acc);
  }
  for (int code = 243; code < 256; ++code) lut_out[code] = nanf("");
  return TQ_OK;
}

tq_status tq_quantize_pack(const void *W_bf16, int64_t n, int64_t k,
                           int32_t group, int32_t planes, uint8_t *codes_out,
                           uint16_t *scales_out, int32_t *dev_status,
                           void *cuda_stream) {
  if (W_bf16 == nullptr || codes_out == nullptr || scales_out == nullptr)
    return TQ_ERR_INVALID_ARG;
  if (n < 0 || k < 0 || planes < 1 || planes > 2) return TQ_ERR_INVALID_ARG;
  if (group != 64 && group != 128) return TQ_ERR_UNSUPPORTED;
  if (k % group != 0) return TQ_ERR_SHAPE;
  if (!aligned(W_bf16, 16) || !aligned(codes_out, 16) ||
      !aligned(scales_out, 4))
    return TQ_ERR_ALIGNMENT;
  if (dev_status != nullptr && !aligned(dev_status, 4)) return TQ_ERR_ALIGNMENT;
  if (n == 0 || k == 0) return TQ_OK;
  return from_cuda(tq::launch_quantize_pack(
      static_cast<const uint16_t *>(W_bf16), n, k, group, planes, codes_out,
      scales_out, dev_status, static_cast<cudaStream_t>(cuda_stream)));
}

tq_status tq_unpack(const tq_weights *w, void *W_bf16_out, int32_t *dev_status,
                    void *cuda_stream) {
  tq::WeightsView v;
  const tq_status st = check_weights(w, &v);
  if (st != TQ_OK) return st;
  if (W_bf16_out == nullptr) return TQ_ERR_INVALID_ARG;
  if (!aligned(W_bf16_out, 16)) return TQ_ERR_ALIGNMENT;
  if (dev_status != nullptr && !aligned(dev_status, 4)) return TQ_ERR_ALIGNMENT;
  if (v.n == 0 || v.k == 0) return TQ_OK;
  return from_cuda(tq::launch_unpack(v, static_cast<uint16_t *>(W_bf16_out),
                                     dev_status,
                                     static_cast<cudaStream_t>(cuda_stream)));
}

tq_status tq_encode_b(const void *W_bf16, int64_t n, int64_t k,
                      const float ladder[5], float zeta,
                      int32_t rows_per_scale, uint8_t *codes_out,
                      uint16_t *rho_out, float *alpha_out, int32_t *dev_status,
                      void *cuda_stream) {
  if (W_bf16 == nullptr || ladder == nullptr || codes_out == nullptr ||
      alpha_out == nullptr)
    return TQ_ERR_INVALID_ARG;
  if (n < 0 || k < 0 || rows_per_scale < 0) return TQ_ERR_INVALID_ARG;
  if (rows_per_scale > 0 && rho_out == nullptr) return TQ_ERR_INVALID_ARG;
  if (!(zeta >= 0.0f && zeta <= 1.0f)) return TQ_ERR_INVALID_ARG;
  for (int i = 0; i < 5; ++i)
    if (!(ladder[i] > 0.0f) || isinf(ladder[i])) return TQ_ERR_INVALID_ARG;
  if (k % 16 != 0) return TQ_ERR_SHAPE;
  if (!aligned(W_bf16, 16) || !aligned(codes_out, 16) ||
      !aligned(alpha_out, 4) || (rho_out != nullptr && !aligned(rho_out, 2)))
    return TQ_ERR_ALIGNMENT;
  if (dev_status != nullptr && !aligned(dev_status, 4)) return TQ_ERR_ALIGNMENT;
  return from_cuda(tq::launch_encode_b(
      static_cast<const uint16_t *>(W_bf16), n, k, ladder, zeta,
      rows_per_scale, codes_out, rows_per_scale > 0 ? rho_out : nullptr,
      alpha_out, dev_status, static_cast<cudaStream_t>(cuda_stream)));
}

tq_status tq_linear(const tq_weights *w, const void *x_bf16, int64_t batch,
                    int64_t ldx, float *y, int64_t ldy, void *cuda_stream) {
  tq::WeightsView v;
  const tq_status st = check_weights(w, &v);
  if (st != TQ_OK) return st;
  if (x_bf16 == nullptr || y == nullptr || batch < 1) return TQ_ERR_INVALID_ARG;
  if (ldx < v.k || ldy < v.n) return TQ_ERR_SHAPE;
  if (!aligned(x_bf16, 16) || ldx % 8 != 0) return TQ_ERR_ALIGNMENT;
  if (!aligned(y, 4)) return TQ_ERR_ALIGNMENT;
  if (v.n == 0) return TQ_OK;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  if (v.k == 0) {  // empty sum: y = 0
    return from_cuda(cudaMemset2DAsync(y, (size_t)ldy * sizeof(float), 0,
                                       (size_t)v.n * sizeof(float),
                                       (size_t)batch, stream));
  }
  return from_cuda(tq::launch_linear(
      v, static_cast<const __nv_bfloat16 *>(x_bf16), batch, ldx, y, ldy,
      stream));
}

tq_status tq_pack7(const uint8_t *codes, int64_t n, int64_t k,
                   uint8_t *used_out, int32_t *n_used_out, uint8_t *packed_out,
                   int32_t *dev_status, void *cuda_stream) {
  if (codes == nullptr || used_out == nullptr || n_used_out == nullptr ||
      packed_out == nullptr || n < 0 || k < 0)
    return TQ_ERR_INVALID_ARG;
  if (k % 16 != 0) return TQ_ERR_SHAPE;
  if (!aligned(codes, 16) || !aligned(used_out, 16) ||
      !aligned(n_used_out, 4) || !aligned(packed_out, 2))
    return TQ_ERR_ALIGNMENT;
  if (dev_status != nullptr && !aligned(dev_status, 4)) return TQ_ERR_ALIGNMENT;
  return from_cuda(tq::launch_pack7(codes, n, k, used_out, n_used_out,
                                    packed_out, dev_status,
                                    static_cast<cudaStream_t>(cuda_stream)));
}

tq_status tq_build_lut7(const float lut[256], const uint8_t used[128],
                        float lut7_out[128]) {
  if (lut == nullptr || used == nullptr || lut7_out == nullptr)
    return TQ_ERR_INVALID_ARG;
  for (int i = 0; i < 128; ++i) lut7_out[i] = lut[used[i]];
  return TQ_OK;
}

tq_status tq_linear_experts(const tq_experts *w, const int32_t *ids,
                            int64_t n_tokens, const void *x_bf16, int64_t ldx,
                            float *y, int64_t ldy, int32_t *dev_status,
                            void *cuda_stream) {
  if (w == nullptr || n_tokens < 0) return TQ_ERR_INVALID_ARG;
  if (w->n_experts < 1 || w->n_hot < 0 || w->n_hot > w->n_experts ||
      w->reserved != 0)
    return TQ_ERR_INVALID_ARG;
  if (w->group != 64) return TQ_ERR_UNSUPPORTED;
  if (w->n_rows < 1 || w->k_cols < 64) return TQ_ERR_SHAPE;
  if (w->k_cols % 64 != 0) return TQ_ERR_SHAPE;
  if (w->codes == nullptr || w->scales == nullptr) return TQ_ERR_INVALID_ARG;
  if (w->n_hot > 0 && (w->codes2 == nullptr || w->scales2 == nullptr))
    return TQ_ERR_INVALID_ARG;
  if (!aligned(w->codes, 16) || !aligned(w->scales, 16)) return TQ_ERR_ALIGNMENT;
  if (w->n_hot > 0 && (!aligned(w->codes2, 16) || !aligned(w->scales2, 16)))
    return TQ_ERR_ALIGNMENT;
  if (n_tokens > 65535) return TQ_ERR_UNSUPPORTED;
  if (n_tokens == 0) return TQ_OK;
  if (ids == nullptr || x_bf16 == nullptr || y == nullptr)
    return TQ_ERR_INVALID_ARG;
  if (ldx < w->k_cols || ldy < w->n_rows) return TQ_ERR_SHAPE;
  if (!aligned(ids, 4) || !aligned(x_bf16, 16) || ldx % 8 != 0 ||
      !aligned(y, 4))
    return TQ_ERR_ALIGNMENT;
  if (dev_status != nullptr && !aligned(dev_status, 4)) return TQ_ERR_ALIGNMENT;
  tq::WeightsView v = {};
  v.format = TQ_FMT_A;
  v.group = 64;
  v.planes = w->n_hot > 0 ? 2 : 1;
  v.rps = 0;
  v.n = w->n_rows;
  v.k = w->k_cols;
  v.codes = w->codes;
  v.scales = w->scales;
  v.lut = nullptr;
  v.lut_rows = 0;
  if (!tq::gemv_a_supported(v, 1)) return TQ_ERR_UNSUPPORTED;
  const int64_t groups = w->n_rows * (w->k_cols / 64);
  tq::ExpertsView E = {};
  E.ids = ids;
  E.n_experts = w->n_experts;
  E.n_hot = w->n_hot;
  E.codes = w->codes;
  E.scales = w->scales;
  E.codes2 = w->codes2;
  E.scales2 = w->scales2;
  E.codes_stride = groups * 13;
  E.scales_stride = groups;
  E.ldx = ldx;
  E.ldy = ldy;
  E.status = dev_status;
  return from_cuda(tq::gemv_a_experts(
      v, E, n_tokens, static_cast<const __nv_bfloat16 *>(x_bf16), y,
      static_cast<cudaStream_t>(cuda_stream)));
}

tq_status tq_testing_linear_wait_fault(int32_t withhold_first_arrive,
                                       uint64_t wait_limit_ns) {
  tq::g_test_skip_first_arrive.store(withhold_first_arrive != 0 ? 1 : 0);
  tq::g_test_wait_ns.store(wait_limit_ns);
  return TQ_OK;
}

tq_status tq_testing_force_linear_path(int32_t path) {
  if (path < 0 || path > 3) return TQ_ERR_INVALID_ARG;
  tq::g_test_force_path.store(path);
  return TQ_OK;
}

tq_status tq_testing_tc_split(int32_t ks, int32_t max_clusters) {
  if (ks < 0 || ks > 8 || max_clusters < 0) return TQ_ERR_INVALID_ARG;
  tq::g_test_tc_ks.store(ks);
  tq::g_test_tc_clusters.store(max_clusters);
  return TQ_OK;
}

tq_status tq_testing_tc_self_check(int32_t enable, uint64_t record_out[4],
                                   int32_t reset) {
  tq::g_test_self_check.store(enable != 0 ? 1 : 0);
  if (record_out == nullptr) return TQ_OK;
  return from_cuda(tq::tc_check_record(record_out, reset != 0));
}

tq_status tq_testing_tc_trace(uint64_t *mapped_host_buffer) {
  tq::g_test_trace.store(
      reinterpret_cast<unsigned long long>(mapped_host_buffer));
  return TQ_OK;
}

const char *tq_status_string(tq_status status) {
  switch (status) {
    case TQ_OK: return "TQ_OK";
    case TQ_ERR_INVALID_ARG: return "TQ_ERR_INVALID_ARG: invalid argument";
    case TQ_ERR_SHAPE: return "TQ_ERR_SHAPE: inconsistent shape or stride";
    case TQ_ERR_ALIGNMENT: return "TQ_ERR_ALIGNMENT: misaligned pointer or stride";
    case TQ_ERR_UNSUPPORTED: return "TQ_ERR_UNSUPPORTED: unsupported parameter";
    case TQ_ERR_BAD_CODE: return "TQ_ERR_BAD_CODE: invalid code byte";
    case TQ_ERR_NONFINITE: return "TQ_ERR_NONFINITE: NaN or Inf weight";
    case TQ_ERR_RANGE: return "TQ_ERR_RANGE: group scale overflows fp16";
    case TQ_ERR_TIMEOUT: return "TQ_ERR_TIMEOUT: in-kernel wait timed out";
    case TQ_ERR_CUDA: return "TQ_ERR_CUDA: CUDA error";
  }
  return "unknown tq_status";
}

}  // extern "C"
