// Format A quantize + pack (precisit.com page, "Three values and a shared
// scale" and "Five trits in a byte"; the second plane follows the FUCINA
// README, "The method", fitted to the fp32 residual of the first).
//
// One thread owns one group of G weights. A block stages 128 consecutive
// groups (a contiguous 16 KB span of W for G = 64) into shared memory with
// coalesced 16-byte loads, in a padded layout (G/2 + 1 words per group) so
// that the per-thread walks over a group are bank-conflict free. The packed
// bytes are staged in shared memory and written out coalesced.
//
// Arithmetic, per group, matching the definition bit for bit:
//   S = sum |W_j| in fp64 over ascending j. A bf16 magnitude m (15 bits) shifted
//   left by 45 is the fp64 pattern of |W| * 2^-896 for every finite value
//   (subnormals included), so S is accumulated in that scaled domain with
//   plain DADDs; scaling by a power of two commutes with every rounding here
//   because all partial sums are non-negative and exact while below the
//   smallest fp64 normal. S * 2^(896 - log2 G) is then the exact fp64 mean.
//   s = fp16_RNE(mean) via cvt.rn.f16.f64.
//   t_j != 0  <=>  |W_j| > s/2, compared on the bit patterns: for non-negative
//   floats the order of the patterns is the order of the values, and the
//   low 16 bits of a bf16 widened to fp32 are zero, so |W| > s/2 iff
//   m > (bits(s/2) >> 16).
//   Plane 2: R_j = fp32_RN(W_j - s1 t1_j) (one IEEE subtraction), the same
//   rule applied to R (its fp32 magnitude shifted by 29 gives |R| * 2^-896).
#include "tq_common.cuh"

namespace tq {
namespace {

constexpr int kGroupsPerBlock = 128;

__device__ __forceinline__ double scaled_f64_from_bf16_mag(uint32_t mag15) {
  return __longlong_as_double((long long)((unsigned long long)mag15 << 45));
}

__device__ __forceinline__ double scaled_f64_from_f32_mag(uint32_t mag31) {
  return __longlong_as_double((long long)((unsigned long long)mag31 << 29));
}

template <int G>
__device__ __forceinline__ uint32_t bf16_at(const uint32_t *gw, int j) {
  return (gw[j >> 1] >> ((j & 1) * 16)) & 0xFFFFu;
}

// fp16 scale bits from the scaled fp64 sum; reports range overflow.
template <int G>
__device__ __forceinline__ uint16_t scale_from_sum(double scaled_sum,
                                                   int32_t *status) {
  constexpr double kUnscale = (G == 64) ? 0x1p890 : 0x1p889;  // 2^896 / G
  const __half h = __double2half(scaled_sum * kUnscale);
  const uint16_t bits = __half_as_ushort(h);
  if ((bits & 0x7FFFu) == 0x7C00u) report(status, TQ_ERR_RANGE);
  return bits;
}

template <int G, int PLANES>
__global__ void __launch_bounds__(kGroupsPerBlock)
    quantize_pack_kernel(const uint16_t *__restrict__ W, int64_t total_groups,
                         uint8_t *__restrict__ codes,
                         uint16_t *__restrict__ scales, int32_t *status) {
  constexpr int NB = bytes_per_group(G);
  constexpr int WORDS = G / 2;
  constexpr int STRIDE = WORDS + 1;
  constexpr int CHUNKS = G / 8;  // 16-byte chunks per group
  __shared__ __align__(16) uint32_t sW[kGroupsPerBlock * STRIDE];
  __shared__ __align__(16) uint8_t sC[PLANES][kGroupsPerBlock * NB];

  const int64_t g0 = (int64_t)blockIdx.x * kGroupsPerBlock;
  const int ng = (int)min((int64_t)kGroupsPerBlock, total_groups - g0);

  // Stage the block's contiguous span of W.
  const uint4 *src = reinterpret_cast<const uint4 *>(W + g0 * G);
  for (int c = threadIdx.x; c < ng * CHUNKS; c += blockDim.x) {
    const uint4 v = __ldcs(src + c);  // streamed once
    uint32_t *d = sW + (c / CHUNKS) * STRIDE + (c % CHUNKS) * 4;
    d[0] = v.x;
    d[1] = v.y;
    d[2] = v.z;
    d[3] = v.w;
  }
  __syncthreads();

  const int t = threadIdx.x;
  if (t < ng) {
    const uint32_t *gw = sW + t * STRIDE;
    // ---- plane 1: scale ----
    double sum = 0.0;
    uint32_t maxmag = 0;
#pragma unroll 8
    for (int w = 0; w < WORDS; ++w) {
      const uint32_t v = gw[w];
      const uint32_t lo = v & 0x7FFFu, hi = (v >> 16) & 0x7FFFu;
      sum += scaled_f64_from_bf16_mag(lo);  // element 2w
      sum += scaled_f64_from_bf16_mag(hi);  // element 2w + 1
      maxmag = max(maxmag, max(lo, hi));
    }
    if (maxmag >= 0x7F80u) report(status, TQ_ERR_NONFINITE);
    const uint16_t s1 = scale_from_sum<G>(sum, status);
    scales[g0 + t] = s1;
    const float s1f = __half2float(__ushort_as_half(s1));
    const uint32_t thr1 =
        (s1 & 0x7FFFu) == 0 ? 0xFFFFu : (__float_as_uint(s1f * 0.5f) >> 16);

    // ---- plane 1: trits -> bytes ----
    // A byte of digits d = t + 1 is sum d_i 3^i = 121 + sum t_i 3^i: start
    // from 121 (all trits 0, also the padding) and add +-3^i per non-zero
    // trit. Every index is a compile-time constant (full unroll).
#pragma unroll
    for (int m = 0; m < NB; ++m) {
      int b = 121;
#pragma unroll
      for (int i = 0; i < 5; ++i) {
        const int j = 5 * m + i;
        if (j < G) {
          const uint32_t v = bf16_at<G>(gw, j);
          constexpr int kP3[5] = {1, 3, 9, 27, 81};
          if ((v & 0x7FFFu) > thr1) b += (v & 0x8000u) ? -kP3[i] : kP3[i];
        }
      }
      sC[0][t * NB + m] = (uint8_t)b;
    }

    if constexpr (PLANES == 2) {
      // ---- plane 2: the same rule on R = fp32_RN(W - s1 t1), computed once
      uint32_t rbits[G];
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const uint32_t v = bf16_at<G>(gw, j);
        const float wf = __uint_as_float(v << 16);
        rbits[j] = (v & 0x7FFFu) <= thr1
                       ? __float_as_uint(wf)  // t1 = 0
                       : __float_as_uint(
                             __fsub_rn(wf, (v & 0x8000u) ? -s1f : s1f));
      }
      double sum2 = 0.0;
#pragma unroll
      for (int j = 0; j < G; ++j)
        sum2 += scaled_f64_from_f32_mag(rbits[j] & 0x7FFFFFFFu);
      const uint16_t s2 = scale_from_sum<G>(sum2, status);
      scales[total_groups + g0 + t] = s2;
      const float s2f = __half2float(__ushort_as_half(s2));
      const uint32_t thr2 =
          (s2 & 0x7FFFu) == 0 ? 0xFFFFFFFFu : __float_as_uint(s2f * 0.5f);
#pragma unroll
      for (int m = 0; m < NB; ++m) {
        int b = 121;
#pragma unroll
        for (int i = 0; i < 5; ++i) {
          const int j = 5 * m + i;
          if (j < G) {
            constexpr int kP3[5] = {1, 3, 9, 27, 81};
            const uint32_t r = rbits[j];
            if ((r & 0x7FFFFFFFu) > thr2)
              b += (r & 0x80000000u) ? -kP3[i] : kP3[i];
          }
        }
        sC[PLANES - 1][t * NB + m] = (uint8_t)b;
      }
    }
  }
  __syncthreads();

  // Coalesced write-out of the packed bytes of every plane.
#pragma unroll
  for (int p = 0; p < PLANES; ++p) {
    uint8_t *dst = codes + ((int64_t)p * total_groups + g0) * NB;
    const int bytes = ng * NB;
    if ((reinterpret_cast<uintptr_t>(dst) & 15) == 0 && (bytes & 15) == 0) {
      const uint4 *s4 = reinterpret_cast<const uint4 *>(sC[p]);
      uint4 *d4 = reinterpret_cast<uint4 *>(dst);
      for (int i = threadIdx.x; i < bytes / 16; i += blockDim.x)
        __stcs(d4 + i, s4[i]);
    } else {
      for (int i = threadIdx.x; i < bytes; i += blockDim.x) dst[i] = sC[p][i];
    }
  }
}

template <int G, int PLANES>
cudaError_t launch(const uint16_t *W, int64_t groups, uint8_t *codes,
                   uint16_t *scales, int32_t *status, cudaStream_t stream) {
  const int64_t blocks = (groups + kGroupsPerBlock - 1) / kGroupsPerBlock;
  quantize_pack_kernel<G, PLANES><<<(unsigned)blocks, kGroupsPerBlock, 0,
                                    stream>>>(W, groups, codes, scales, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize_pack(const uint16_t *W, int64_t n, int64_t k,
                                 int G, int planes, uint8_t *codes,
                                 uint16_t *scales, int32_t *status,
                                 cudaStream_t stream) {
  const int64_t groups = n * (k / G);
  if (G == 64) {
    return planes == 1 ? launch<64, 1>(W, groups, codes, scales, status, stream)
                       : launch<64, 2>(W, groups, codes, scales, status, stream);
  }
  return planes == 1 ? launch<128, 1>(W, groups, codes, scales, status, stream)
                     : launch<128, 2>(W, groups, codes, scales, status, stream);
}

}  // namespace tq
