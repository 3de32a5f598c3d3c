// 7-bit truncated alphabet ("A Discrete Weight Language for Large Language
// Models", alphaneural.io, section 8.1 "Variable-depth words"): a layer that
// uses at most 128 of the 243 words stores, per weight, the 7-bit index of
// its code in the layer's table of used codes (ascending), 16 indices per
// 14 bytes, little-endian (index j at bits 7j .. 7j + 6 of the chunk).
//
// Packing runs in three launches and keeps its intermediate state in its
// own output `used` (128 bytes): the first 32 bytes hold the 256-bit set of
// codes present while it is gathered.
//   1. mark: every thread reads 16 codes, sets their bits in a per-CTA set
//      (shared memory), merged into the output's set (atomic OR);
//   2. list: one CTA turns the set into the ascending table, pads it with
//      the all-zero word 121 and writes the count (more than 128 words is
//      TQ_ERR_RANGE);
//   3. pack: every thread turns 16 codes into 16 indices (inverse table in
//      shared memory) and writes their 14 bytes as 7 aligned 2-byte words.
// Decoding index i gives LUT7[i] = LUT[used[i]] (tq_build_lut7).
#include "tq_common.cuh"
#include "tq_linear.cuh"

namespace tq {
namespace {

__global__ void __launch_bounds__(256)
    pack7_mark_kernel(const uint4 *__restrict__ codes, int64_t chunks,
                      uint32_t *set) {
  __shared__ uint32_t s[8];
  if (threadIdx.x < 8) s[threadIdx.x] = 0;
  __syncthreads();
  for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < chunks;
       c += (int64_t)gridDim.x * blockDim.x) {
    const uint4 v = __ldg(codes + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t b = (w[i >> 2] >> (8 * (i & 3))) & 0xFFu;
      atomicOr(&s[b >> 5], 1u << (b & 31));
    }
  }
  __syncthreads();
  if (threadIdx.x < 8 && s[threadIdx.x] != 0)
    atomicOr(set + threadIdx.x, s[threadIdx.x]);
}

__global__ void __launch_bounds__(256)
    pack7_list_kernel(uint8_t *used, int32_t *n_used, int32_t *status) {
  __shared__ uint32_t s[8];
  __shared__ int warp_count[8];
  const int c = threadIdx.x;  // one thread per code value
  if (c < 8) s[c] = reinterpret_cast<const uint32_t *>(used)[c];
  __syncthreads();  // the set is read before the table overwrites it
  const bool present = (s[c >> 5] >> (c & 31)) & 1u;
  const uint32_t ballot = __ballot_sync(0xFFFFFFFFu, present);
  const int lane = c & 31, warp = c >> 5;
  if (lane == 0) warp_count[warp] = __popc(ballot);
  __syncthreads();
  int before = 0, total = 0;
  for (int i = 0; i < 8; ++i) {
    before += i < warp ? warp_count[i] : 0;
    total += warp_count[i];
  }
  const int idx = before + __popc(ballot & ((1u << lane) - 1u));
  if (c < 128 && c >= total) used[c] = 121;  // padding: the all-zero word
  if (present && idx < 128) used[idx] = (uint8_t)c;
  if (c == 0) {
    *n_used = total;
    if (total > 128) report(status, TQ_ERR_RANGE);
  }
}

__global__ void __launch_bounds__(256)
    pack7_kernel(const uint4 *__restrict__ codes, int64_t chunks,
                 const uint8_t *__restrict__ used, uint16_t *__restrict__ out) {
  __shared__ uint8_t index_of[256];
  index_of[threadIdx.x] = 0;
  __syncthreads();
  if (threadIdx.x < 128) {
    // the table is ascending; its padding (121) may repeat a real word
    // only past the count, where the first entry already holds it
    const uint8_t c = used[threadIdx.x];
    if (threadIdx.x == 0 || used[threadIdx.x - 1] < c) index_of[c] = threadIdx.x;
  }
  __syncthreads();
  for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < chunks;
       c += (int64_t)gridDim.x * blockDim.x) {
    const uint4 v = __ldg(codes + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint64_t lo = 0, hi = 0;  // bits 0..63 and 64..111 of the chunk
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint64_t idx = index_of[(w[j >> 2] >> (8 * (j & 3))) & 0xFFu];
      const int pos = 7 * j;
      if (pos < 64) lo |= idx << pos;
      if (pos + 7 > 64) hi |= pos >= 64 ? idx << (pos - 64) : idx >> (64 - pos);
    }
    uint16_t *o = out + 7 * c;
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = (uint16_t)(lo >> (16 * i));
#pragma unroll
    for (int i = 0; i < 3; ++i) o[4 + i] = (uint16_t)(hi >> (16 * i));
  }
}

}  // namespace

cudaError_t launch_pack7(const uint8_t *codes, int64_t n, int64_t k,
                         uint8_t *used, int32_t *n_used, uint8_t *packed,
                         int32_t *status, cudaStream_t stream) {
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if ((e = cudaMemsetAsync(used, 0, 128, stream)) != cudaSuccess) return e;
  const int64_t chunks = n * (k / 16);
  const int64_t want = (chunks + 255) / 256;
  const int grid = (int)(want < 8LL * sms ? (want > 0 ? want : 1) : 8LL * sms);
  pack7_mark_kernel<<<grid, 256, 0, stream>>>(
      reinterpret_cast<const uint4 *>(codes), chunks,
      reinterpret_cast<uint32_t *>(used));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  pack7_list_kernel<<<1, 256, 0, stream>>>(used, n_used, status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (chunks == 0) return cudaSuccess;
  pack7_kernel<<<grid, 256, 0, stream>>>(
      reinterpret_cast<const uint4 *>(codes), chunks, used,
      reinterpret_cast<uint16_t *>(packed));
  return cudaGetLastError();
}

}  // namespace tq
