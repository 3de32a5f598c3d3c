// Reference-structure fused matmul: one warp per output row, decode in
// registers, fp32 accumulation, warp-shuffle reduction. Plain and general
// (any G, planes, batch tile of 1..8, unaligned Format A groups); the tuned
// kernels are checked against the same oracle and replace it where they
// apply.
//
//   Format A: y[b][n] = sum_p sum_g s_p[n][g] * sum_{j in g} t_p[n][j] x[b][j]
//   Format B: y[b][n] = rho[n / rps] * sum_k LUT[code[n][k]] x[b][k]
#include "tq_common.cuh"
#include "tq_linear.cuh"

namespace tq {
namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &v, float *f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    f[2 * q] = __uint_as_float(w[q] << 16);
    f[2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
  }
}

// One warp per row. The code book sits in shared memory: the layer's one
// book, or with one book per block of lut_rows rows (adaptive alphabet)
// each warp's copy of its row's book.
template <int BT>
__global__ void __launch_bounds__(kWarps * 32)
    linear_b_simple(const uint8_t *__restrict__ codes, int64_t n, int64_t k,
                    const float *__restrict__ lut, int64_t lut_rows,
                    const uint16_t *__restrict__ rho, int rps,
                    const __nv_bfloat16 *__restrict__ x, int64_t ldx,
                    float *__restrict__ y, int64_t ldy) {
  __shared__ float sLw[kWarps][kLutEntries];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t row = (int64_t)blockIdx.x * kWarps + warp;
  if (row >= n) return;
  float *sL = sLw[warp];
  const float *rl = lut_rows > 0 ? lut + (row / lut_rows) * kLutEntries : lut;
  for (int i = lane; i < kLutEntries; i += 32) sL[i] = rl[i];
  __syncwarp();
  float acc[BT];
#pragma unroll
  for (int b = 0; b < BT; ++b) acc[b] = 0.0f;
  const uint8_t *cr = codes + row * k;
  for (int64_t c = lane * 16; c < k; c += 512) {
    const uint4 cv = *reinterpret_cast<const uint4 *>(cr + c);
    const uint32_t cw[4] = {cv.x, cv.y, cv.z, cv.w};
    float wv[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) wv[e] = sL[(cw[e / 4] >> (8 * (e % 4))) & 0xFF];
#pragma unroll
    for (int b = 0; b < BT; ++b) {
      const uint4 *xp = reinterpret_cast<const uint4 *>(x + b * ldx + c);
      float xv[16];
      bf16x8_to_f32(xp[0], xv);
      bf16x8_to_f32(xp[1], xv + 8);
#pragma unroll
      for (int e = 0; e < 16; ++e) acc[b] = fmaf(wv[e], xv[e], acc[b]);
    }
  }
  const float r = rho ? __half2float(__ushort_as_half(rho[row / rps])) : 1.0f;
#pragma unroll
  for (int b = 0; b < BT; ++b) {
    const float s = warp_sum(acc[b]);
    if (lane == 0) y[b * ldy + row] = r * s;
  }
}

// 7-bit alphabet: one warp per row, lane chunks of 16 indices (14 bytes);
// weights LUT7[i] (times rho on the accumulator, as Format B).
template <int BT>
__global__ void __launch_bounds__(kWarps * 32)
    linear_b7_simple(const uint16_t *__restrict__ packed, int64_t n, int64_t k,
                     const float *__restrict__ lut7,
                     const uint16_t *__restrict__ rho, int rps,
                     const __nv_bfloat16 *__restrict__ x, int64_t ldx,
                     float *__restrict__ y, int64_t ldy) {
  __shared__ float sL[128];
  if (threadIdx.x < 128) sL[threadIdx.x] = lut7[threadIdx.x];
  __syncthreads();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t row = (int64_t)blockIdx.x * kWarps + warp;
  if (row >= n) return;
  float acc[BT];
#pragma unroll
  for (int b = 0; b < BT; ++b) acc[b] = 0.0f;
  const int64_t cpr = k / 16;
  const uint16_t *pr = packed + row * cpr * 7;
  for (int64_t ch = lane; ch < cpr; ch += 32) {
    uint32_t idx[16];
    unpack7_chunk(pr + 7 * ch, idx);
    float wv[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) wv[e] = sL[idx[e]];
#pragma unroll
    for (int b = 0; b < BT; ++b) {
      const uint4 *xp = reinterpret_cast<const uint4 *>(x + b * ldx + 16 * ch);
      float xv[16];
      bf16x8_to_f32(xp[0], xv);
      bf16x8_to_f32(xp[1], xv + 8);
#pragma unroll
      for (int e = 0; e < 16; ++e) acc[b] = fmaf(wv[e], xv[e], acc[b]);
    }
  }
  const float r = rho ? __half2float(__ushort_as_half(rho[row / rps])) : 1.0f;
#pragma unroll
  for (int b = 0; b < BT; ++b) {
    const float s = warp_sum(acc[b]);
    if (lane == 0) y[b * ldy + row] = r * s;
  }
}

template <int G, int PLANES, int BT>
__global__ void __launch_bounds__(kWarps * 32)
    linear_a_simple(const uint8_t *__restrict__ codes,
                    const uint16_t *__restrict__ scales, int64_t n, int64_t k,
                    int64_t cps, int64_t sps,
                    const __nv_bfloat16 *__restrict__ x, int64_t ldx,
                    float *__restrict__ y, int64_t ldy) {
  constexpr int NB = bytes_per_group(G);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t row = (int64_t)blockIdx.x * kWarps + warp;
  if (row >= n) return;
  const int64_t gpr = k / G;
  float acc[BT];
#pragma unroll
  for (int b = 0; b < BT; ++b) acc[b] = 0.0f;
  for (int64_t g = lane; g < gpr; g += 32) {
#pragma unroll
    for (int p = 0; p < PLANES; ++p) {
      const int64_t gi = row * gpr + g;
      const uint8_t *cb = codes + p * cps + gi * NB;
      const float s = __half2float(__ushort_as_half(scales[p * sps + gi]));
      float part[BT];
#pragma unroll
      for (int b = 0; b < BT; ++b) part[b] = 0.0f;
      for (int m = 0; m < NB; ++m) {
        uint32_t byte = cb[m];
#pragma unroll
        for (int i = 0; i < 5; ++i) {
          const int j = 5 * m + i;
          const uint32_t d = byte % 3u;
          byte /= 3u;
          if (j < G && d != 1u) {
#pragma unroll
            for (int b = 0; b < BT; ++b) {
              const float xv = __bfloat162float(x[b * ldx + g * G + j]);
              part[b] = (d == 2u) ? part[b] + xv : part[b] - xv;
            }
          }
        }
      }
#pragma unroll
      for (int b = 0; b < BT; ++b) acc[b] = fmaf(s, part[b], acc[b]);
    }
  }
#pragma unroll
  for (int b = 0; b < BT; ++b) {
    const float s = warp_sum(acc[b]);
    if (lane == 0) y[b * ldy + row] = s;
  }
}

template <int BT>
cudaError_t launch_b(const WeightsView &w, const __nv_bfloat16 *x, int64_t ldx,
                     float *y, int64_t ldy, cudaStream_t stream) {
  const unsigned blocks = (unsigned)((w.n + kWarps - 1) / kWarps);
  linear_b_simple<BT><<<blocks, kWarps * 32, 0, stream>>>(
      w.codes, w.n, w.k, w.lut, w.lut_rows, w.scales, w.rps, x, ldx, y, ldy);
  return cudaGetLastError();
}

template <int G, int PLANES, int BT>
cudaError_t launch_a(const WeightsView &w, const __nv_bfloat16 *x, int64_t ldx,
                     float *y, int64_t ldy, cudaStream_t stream) {
  const unsigned blocks = (unsigned)((w.n + kWarps - 1) / kWarps);
  linear_a_simple<G, PLANES, BT><<<blocks, kWarps * 32, 0, stream>>>(
      w.codes, w.scales, w.n, w.k, w.codes_plane_stride, w.scales_plane_stride,
      x, ldx, y, ldy);
  return cudaGetLastError();
}

template <int BT>
cudaError_t launch_tile(const WeightsView &w, const __nv_bfloat16 *x,
                        int64_t ldx, float *y, int64_t ldy,
                        cudaStream_t stream) {
  if (w.format == TQ_FMT_B) return launch_b<BT>(w, x, ldx, y, ldy, stream);
  if (w.format == TQ_FMT_B7) {
    const unsigned blocks = (unsigned)((w.n + kWarps - 1) / kWarps);
    linear_b7_simple<BT><<<blocks, kWarps * 32, 0, stream>>>(
        reinterpret_cast<const uint16_t *>(w.codes), w.n, w.k, w.lut,
        w.scales, w.rps, x, ldx, y, ldy);
    return cudaGetLastError();
  }
  if (w.group == 64)
    return w.planes == 1 ? launch_a<64, 1, BT>(w, x, ldx, y, ldy, stream)
                         : launch_a<64, 2, BT>(w, x, ldx, y, ldy, stream);
  return w.planes == 1 ? launch_a<128, 1, BT>(w, x, ldx, y, ldy, stream)
                       : launch_a<128, 2, BT>(w, x, ldx, y, ldy, stream);
}

}  // namespace

cudaError_t linear_simple(const WeightsView &w, const __nv_bfloat16 *x,
                          int64_t batch, int64_t ldx, float *y, int64_t ldy,
                          cudaStream_t stream) {
  for (int64_t b0 = 0; b0 < batch; b0 += 8) {
    const int bt = (int)(batch - b0 < 8 ? batch - b0 : 8);
    const __nv_bfloat16 *xb = x + b0 * ldx;
    float *yb = y + b0 * ldy;
    cudaError_t e;
    switch (bt) {
      case 1: e = launch_tile<1>(w, xb, ldx, yb, ldy, stream); break;
      case 2: e = launch_tile<2>(w, xb, ldx, yb, ldy, stream); break;
      case 3: e = launch_tile<3>(w, xb, ldx, yb, ldy, stream); break;
      case 4: e = launch_tile<4>(w, xb, ldx, yb, ldy, stream); break;
      case 5: e = launch_tile<5>(w, xb, ldx, yb, ldy, stream); break;
      case 6: e = launch_tile<6>(w, xb, ldx, yb, ldy, stream); break;
      case 7: e = launch_tile<7>(w, xb, ldx, yb, ldy, stream); break;
      default: e = launch_tile<8>(w, xb, ldx, yb, ldy, stream); break;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace tq
