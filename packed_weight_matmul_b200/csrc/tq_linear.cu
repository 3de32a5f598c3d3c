// Dispatch of tq_linear to the fused matmul kernels.
#include "tq_linear.cuh"

namespace tq {

std::atomic<int> g_test_force_path{0};

cudaError_t launch_linear(const WeightsView &w, const __nv_bfloat16 *x,
                          int64_t batch, int64_t ldx, float *y, int64_t ldy,
                          cudaStream_t stream) {
  const int force = g_test_force_path.load();
  if ((force == 2 || force == 3) && gemm_tc_supported(w, batch))
    return gemm_tc(w, x, batch, ldx, y, ldy, stream);
  if (w.format == TQ_FMT_B7) {
    // 7-bit indices: the tensor-core kernel from batch 3 when K is a
    // multiple of 128 (at 8192 x 5376 it runs in 33 us at batches 1-8; the
    // one-warp-per-row kernel takes 30 us at batch 2, 36 us at batch 3),
    // else the one-warp-per-row kernel
    if (force != 1 && batch >= 3 && gemm_tc_supported(w, batch))
      return gemm_tc(w, x, batch, ldx, y, ldy, stream);
    return linear_simple(w, x, batch, ldx, y, ldy, stream);
  }
  if (w.format == TQ_FMT_B && w.lut_rows > 0) {
    // adaptive alphabet: the tensor-core kernel when every warp's 32 rows
    // share a code book (any batch), else the one-warp-per-row kernel
    if (gemm_tc_supported(w, batch))
      return gemm_tc(w, x, batch, ldx, y, ldy, stream);
    return linear_simple(w, x, batch, ldx, y, ldy, stream);
  }
  if (force == 1) {
    if (gemv_b_supported(w, batch))
      return gemv_b(w, x, batch, ldx, y, ldy, stream);
    if (gemv_a_supported(w, batch)) return gemv_a(w, x, y, stream);
    return linear_simple(w, x, batch, ldx, y, ldy, stream);
  }
  if (gemv_b_supported(w, batch))
    return gemv_b(w, x, batch, ldx, y, ldy, stream);
  if (gemv_a_supported(w, batch)) return gemv_a(w, x, y, stream);
  const int64_t tc_min_batch = w.format == TQ_FMT_B ? 5 : 2;
  if (batch >= tc_min_batch && gemm_tc_supported(w, batch))
    return gemm_tc(w, x, batch, ldx, y, ldy, stream);
  return linear_simple(w, x, batch, ldx, y, ldy, stream);
}

}  // namespace tq
