// Decode a package to bf16, validating every code byte.
//
// Format A (precisit.com page, "Three values and a shared scale" and "Five
// trits in a byte"): W_hat = bf16_RNE(fp32_RN(s1 t1 [+ s2 t2])); a byte >= 243
// or a padding digit other than 1 is TQ_ERR_BAD_CODE.
// Format B (alphaneural.io page, sections 3.2-3.3): W_hat =
// bf16_RNE(fp32_RN(rho * LUT[code])) or bf16_RNE(LUT[code]); a code >= 243 is
// TQ_ERR_BAD_CODE.
//
// This is the validation and cross-check path, not the matmul: it writes the
// bf16 matrix the fused kernels never materialise.
#include "tq_common.cuh"

namespace tq {
namespace {

constexpr int kGroupsPerBlock = 128;

// Copy `bytes` bytes from global `src` to shared `dst` (16-byte vectors when
// both ends allow it).
__device__ __forceinline__ void stage_bytes(uint8_t *dst, const uint8_t *src,
                                            int bytes) {
  if ((reinterpret_cast<uintptr_t>(src) & 15) == 0 && (bytes & 15) == 0) {
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
    for (int i = threadIdx.x; i < bytes / 16; i += blockDim.x) d4[i] = __ldcs(s4 + i);
  } else {
    for (int i = threadIdx.x; i < bytes; i += blockDim.x) dst[i] = __ldcs(src + i);
  }
}

template <int G, int PLANES>
__global__ void __launch_bounds__(kGroupsPerBlock)
    unpack_a_kernel(const uint8_t *__restrict__ codes,
                    const uint16_t *__restrict__ scales, int64_t total_groups,
                    int64_t codes_plane_stride, int64_t scales_plane_stride,
                    uint16_t *__restrict__ out, int32_t *status) {
  constexpr int NB = bytes_per_group(G);
  constexpr int STRIDE_H = G + 2;  // half-words per staged output group
  __shared__ __align__(16) uint8_t sC[PLANES][kGroupsPerBlock * NB + 16];
  __shared__ __align__(16) uint16_t sO[kGroupsPerBlock * STRIDE_H];

  const int64_t g0 = (int64_t)blockIdx.x * kGroupsPerBlock;
  const int ng = (int)min((int64_t)kGroupsPerBlock, total_groups - g0);
#pragma unroll
  for (int p = 0; p < PLANES; ++p)
    stage_bytes(sC[p], codes + p * codes_plane_stride + g0 * NB, ng * NB);
  __syncthreads();

  const int t = threadIdx.x;
  if (t < ng) {
    float s[PLANES];
#pragma unroll
    for (int p = 0; p < PLANES; ++p)
      s[p] = __half2float(__ushort_as_half(
          scales[p * scales_plane_stride + g0 + t]));
    bool bad = false;
#pragma unroll 1
    for (int m = 0; m < NB; ++m) {
      uint32_t b[PLANES];
#pragma unroll
      for (int p = 0; p < PLANES; ++p) {
        b[p] = sC[p][t * NB + m];
        bad |= b[p] >= 243u;
      }
#pragma unroll
      for (int i = 0; i < 5; ++i) {
        const int j = 5 * m + i;
        float v = 0.0f;
#pragma unroll
        for (int p = 0; p < PLANES; ++p) {
          const uint32_t d = b[p] % 3u;
          b[p] /= 3u;
          if (j < G) {
            // s * t is exact in fp32; the plane sum is one fp32 rounding.
            const float st = (d == 1u) ? 0.0f : (d == 2u ? s[p] : -s[p]);
            v = (p == 0) ? st : __fadd_rn(v, st);
          } else {
            bad |= d != 1u;  // padding must decode to zero
          }
        }
        if (j < G)
          sO[t * STRIDE_H + j] =
              __bfloat16_as_ushort(__float2bfloat16_rn(v));
      }
    }
    if (bad) report(status, TQ_ERR_BAD_CODE);
  }
  __syncthreads();

  // Coalesced write-out: ng * G bf16, contiguous in the output.
  uint32_t *dst = reinterpret_cast<uint32_t *>(out + g0 * G);
  const uint32_t *src32 = reinterpret_cast<const uint32_t *>(sO);
  for (int i = threadIdx.x; i < ng * (G / 2); i += blockDim.x) {
    const int g = i / (G / 2), w = i % (G / 2);
    __stcs(dst + i, src32[g * (STRIDE_H / 2) + w]);
  }
}

// Format B: one thread per 16 codes (k % 16 == 0, so a chunk never crosses a
// row). With one code book per block of lut_rows rows (adaptive alphabet)
// the row's book is read through the read-only cache.
__global__ void __launch_bounds__(256)
    unpack_b_kernel(const uint8_t *__restrict__ codes, int64_t n, int64_t k,
                    const float *__restrict__ lut, int64_t lut_rows,
                    const uint16_t *__restrict__ rho, int rps,
                    uint16_t *__restrict__ out, int32_t *status) {
  __shared__ float sL[kLutEntries];
  for (int i = threadIdx.x; i < kLutEntries; i += blockDim.x) sL[i] = lut[i];
  __syncthreads();
  const int64_t chunks = n * (k / 16);
  bool bad = false;
  for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < chunks;
       c += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = (c * 16) / k;
    const float r = rho ? __half2float(__ushort_as_half(rho[row / rps])) : 1.0f;
    const float *rl = lut_rows > 0 ? lut + (row / lut_rows) * kLutEntries : nullptr;
    const uint4 cv = __ldcs(reinterpret_cast<const uint4 *>(codes) + c);
    const uint32_t words[4] = {cv.x, cv.y, cv.z, cv.w};
    uint32_t o[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint16_t h[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t code = (words[q] >> (8 * e)) & 0xFFu;
        bad |= code >= 243u;
        float v = rl != nullptr ? __ldg(rl + code) : sL[code];
        if (rho) v = __fmul_rn(r, v);  // fp16 x fp32 rounded once to fp32
        h[e] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
      }
      o[2 * q] = h[0] | ((uint32_t)h[1] << 16);
      o[2 * q + 1] = h[2] | ((uint32_t)h[3] << 16);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(out) + 2 * c;
    __stcs(dst, make_uint4(o[0], o[1], o[2], o[3]));
    __stcs(dst + 1, make_uint4(o[4], o[5], o[6], o[7]));
  }
  if (bad) report(status, TQ_ERR_BAD_CODE);
}

// 7-bit alphabet: one thread per 16 indices (14 bytes); index i decodes to
// LUT7[i] = LUT[used[i]] (times rho), exactly Format B's weight.
__global__ void __launch_bounds__(256)
    unpack_b7_kernel(const uint16_t *__restrict__ packed, int64_t chunks,
                     int64_t chunks_per_row, const float *__restrict__ lut7,
                     const uint16_t *__restrict__ rho, int rps,
                     uint16_t *__restrict__ out) {
  __shared__ float sL[128];
  if (threadIdx.x < 128) sL[threadIdx.x] = lut7[threadIdx.x];
  __syncthreads();
  for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < chunks;
       c += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = c / chunks_per_row;
    const float r = rho ? __half2float(__ushort_as_half(rho[row / rps])) : 1.0f;
    uint32_t idx[16];
    unpack7_chunk(packed + 7 * c, idx);
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float v0 = sL[idx[2 * j]], v1 = sL[idx[2 * j + 1]];
      if (rho) {
        v0 = __fmul_rn(r, v0);
        v1 = __fmul_rn(r, v1);
      }
      o[j] = __bfloat16_as_ushort(__float2bfloat16_rn(v0)) |
             ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v1)) << 16);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(out) + 2 * c;
    __stcs(dst, make_uint4(o[0], o[1], o[2], o[3]));
    __stcs(dst + 1, make_uint4(o[4], o[5], o[6], o[7]));
  }
}

template <int G, int PLANES>
cudaError_t launch_a(const WeightsView &w, uint16_t *out, int32_t *status,
                     cudaStream_t stream) {
  const int64_t groups = w.n * (w.k / G);
  const int64_t blocks = (groups + kGroupsPerBlock - 1) / kGroupsPerBlock;
  unpack_a_kernel<G, PLANES><<<(unsigned)blocks, kGroupsPerBlock, 0, stream>>>(
      w.codes, w.scales, groups, w.codes_plane_stride, w.scales_plane_stride,
      out, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_unpack(const WeightsView &w, uint16_t *out,
                          int32_t *status, cudaStream_t stream) {
  if (w.format == TQ_FMT_A) {
    if (w.group == 64)
      return w.planes == 1 ? launch_a<64, 1>(w, out, status, stream)
                           : launch_a<64, 2>(w, out, status, stream);
    return w.planes == 1 ? launch_a<128, 1>(w, out, status, stream)
                         : launch_a<128, 2>(w, out, status, stream);
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t chunks = w.n * (w.k / 16);
  const int64_t want = (chunks + 255) / 256;
  const int blocks = (int)(want < (int64_t)sms * 8 ? want : (int64_t)sms * 8);
  if (w.format == TQ_FMT_B7) {
    unpack_b7_kernel<<<blocks, 256, 0, stream>>>(
        reinterpret_cast<const uint16_t *>(w.codes), chunks, w.k / 16, w.lut,
        w.scales, w.rps, out);
    return cudaGetLastError();
  }
  unpack_b_kernel<<<blocks, 256, 0, stream>>>(
      w.codes, w.n, w.k, w.lut, w.lut_rows, w.scales, w.rps, out, status);
  return cudaGetLastError();
}

}  // namespace tq
