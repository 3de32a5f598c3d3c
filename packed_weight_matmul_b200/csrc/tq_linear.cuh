// Internal interface of the fused matmul kernels and their dispatcher.
#pragma once

#include "tq_common.cuh"

namespace tq {

// Test hooks of the tensor-core kernel (tq_testing.h).
extern std::atomic<uint64_t> g_test_wait_ns;
extern std::atomic<int> g_test_skip_first_arrive;
// Kernel family forced by tq_testing_force_linear_path (0 = automatic).
extern std::atomic<int> g_test_force_path;
// Self-checking tensor-core kernel (tq_testing_tc_self_check) and its record.
extern std::atomic<int> g_test_self_check;
extern std::atomic<unsigned long long> g_test_trace;
// Split of K and cluster cap forced by tq_testing_tc_split (0 = automatic).
extern std::atomic<int> g_test_tc_ks;
extern std::atomic<int> g_test_tc_clusters;
cudaError_t tc_check_record(uint64_t out[4], bool reset);

// One warp per row; any shape the boundary accepts.
cudaError_t linear_simple(const WeightsView &w, const __nv_bfloat16 *x,
                          int64_t batch, int64_t ldx, float *y, int64_t ldy,
                          cudaStream_t stream);

// Format B, batch 1..4: CUDA-core GEMV with a replicated code book.
bool gemv_b_supported(const WeightsView &w, int64_t batch);
cudaError_t gemv_b(const WeightsView &w, const __nv_bfloat16 *x, int64_t batch,
                   int64_t ldx, float *y, int64_t ldy, cudaStream_t stream);

// Format A, batch 1, G = 64: activation tables (243 partial sums of x per
// code byte position), one table load per code byte.
bool gemv_a_supported(const WeightsView &w, int64_t batch);
cudaError_t gemv_a(const WeightsView &w, const __nv_bfloat16 *x, float *y,
                   cudaStream_t stream);
// Expert-indexed batch-1 GEMVs (tq_linear_experts): `w` describes one
// expert's matrix (n, k, group); token t multiplies x row t by expert
// E.ids[t] into y row t.
cudaError_t gemv_a_experts(const WeightsView &w, const ExpertsView &E,
                           int64_t tokens, const __nv_bfloat16 *x, float *y,
                           cudaStream_t stream);
// 7-bit truncated alphabet: used-code table and packed indices of codes.
cudaError_t launch_pack7(const uint8_t *codes, int64_t n, int64_t k,
                         uint8_t *used, int32_t *n_used, uint8_t *packed,
                         int32_t *status, cudaStream_t stream);

// Batches that are a real contraction: tcgen05 MMAs on decoded bf16 hi/lo
// operands, accumulator in tensor memory.
bool gemm_tc_supported(const WeightsView &w, int64_t batch);
cudaError_t gemm_tc(const WeightsView &w, const __nv_bfloat16 *x,
                    int64_t batch, int64_t ldx, float *y, int64_t ldy,
                    cudaStream_t stream);

}  // namespace tq
