// Shared declarations of the tq CUDA library (sm_100a).
#pragma once

#include <atomic>
#include <utility>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tq.h"

namespace tq {

constexpr int kLutEntries = 256;  // 243 words + NaN padding

__host__ __device__ constexpr int bytes_per_group(int G) { return (G + 4) / 5; }

// First error wins: the status word moves away from TQ_OK only once.
__device__ __forceinline__ void report(int32_t *status, int code) {
  if (status != nullptr) atomicCAS(status, (int32_t)TQ_OK, (int32_t)code);
}

// Validated, flattened view of a tq_weights descriptor.
struct WeightsView {
  int format;
  int group;
  int planes;
  int rps;
  int64_t n, k;
  const uint8_t *codes;
  const uint16_t *scales;  // A: group scales; B: rho or nullptr
  const float *lut;
  int64_t codes_plane_stride;   // bytes
  int64_t scales_plane_stride;  // elements
  int64_t lut_rows;             // B: rows per code book (0: one for all)
};

// 7-bit alphabet: the 16 indices of a 14-byte chunk (7 aligned 2-byte words,
// index j at bits 7j .. 7j + 6, little-endian).
__device__ __forceinline__ void unpack7_chunk(const uint16_t *__restrict__ p,
                                              uint32_t (&idx)[16]) {
  uint64_t lo = 0, hi = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) lo |= (uint64_t)__ldg(p + i) << (16 * i);
#pragma unroll
  for (int i = 0; i < 3; ++i) hi |= (uint64_t)__ldg(p + 4 + i) << (16 * i);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int pos = 7 * j;
    uint64_t v;
    if (pos + 7 <= 64)
      v = lo >> pos;
    else if (pos >= 64)
      v = hi >> (pos - 64);
    else
      v = (lo >> pos) | (hi << (64 - pos));
    idx[j] = (uint32_t)v & 0x7Fu;
  }
}

// Expert-indexed Format A call (tq_linear_experts): token t uses expert
// ids[t]; ids == nullptr marks a plain call.
struct ExpertsView {
  const int32_t *ids;
  int n_experts, n_hot;
  const uint8_t *codes;    // plane 1 of every expert
  const uint16_t *scales;
  const uint8_t *codes2;   // plane 2 of experts 0 .. n_hot - 1
  const uint16_t *scales2;
  int64_t codes_stride;    // bytes between experts
  int64_t scales_stride;   // elements between experts
  int64_t ldx, ldy;
  int32_t *status;
};

// Programmatic dependent launch. A kernel launched with programmatic stream
// serialization may start while the kernel before it on the stream is still
// running (once every CTA of that kernel has called pdl_launch_dependents or
// exited). Before pdl_wait it may only touch its own shared memory and
// tensor memory and hint the L2 cache (prefetches do not read into the SM,
// and L2 is coherent, so a prefetch of bytes the earlier kernel is still
// writing is harmless); pdl_wait returns once the earlier kernel has
// completed and its writes are visible, so every read of user memory and
// every global write comes after it. Without the attribute pdl_wait returns
// at once.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// L2 prefetch of `bytes` (a multiple of 16, 16-byte aligned) at `p`.
__device__ __forceinline__ void prefetch_l2_bulk(const void *p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p),
               "r"(bytes)
               : "memory");
}

// Launch `kern` with programmatic stream serialization (see pdl_wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block,
                       size_t smem, cudaStream_t stream, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Raise a kernel's dynamic shared-memory limit to `bytes` once per device.
// The attribute is one value per function and context; every caller asks for
// the same (largest) value, so concurrent callers cannot lower it under one
// another's launch. Occupancy follows each launch's own request.
template <auto Kern>
cudaError_t ensure_smem_limit(int bytes) {
  static std::atomic<uint64_t> done{0};  // bit d: set on device d (< 64)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? 1ull << dev : 0ull;
  if (bit != 0 && (done.load(std::memory_order_acquire) & bit) != 0)
    return cudaSuccess;
  e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           bytes);
  if (e == cudaSuccess && bit != 0)
    done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// ---- launchers (each enqueues on `stream`, returns the launch error) ----
cudaError_t launch_quantize_pack(const uint16_t *W, int64_t n, int64_t k,
                                 int G, int planes, uint8_t *codes,
                                 uint16_t *scales, int32_t *status,
                                 cudaStream_t stream);
cudaError_t launch_unpack(const WeightsView &w, uint16_t *out,
                          int32_t *status, cudaStream_t stream);
cudaError_t launch_encode_b(const uint16_t *W, int64_t n, int64_t k,
                            const float ladder[5], float zeta, int rps,
                            uint8_t *codes, uint16_t *rho, float *alpha,
                            int32_t *status, cudaStream_t stream);
cudaError_t launch_linear(const WeightsView &w, const __nv_bfloat16 *x,
                          int64_t batch, int64_t ldx, float *y, int64_t ldy,
                          cudaStream_t stream);

}  // namespace tq
