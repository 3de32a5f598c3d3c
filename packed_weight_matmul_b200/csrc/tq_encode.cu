// Format B encoder ("A Discrete Weight Language for Large Language Models",
// alphaneural.io, section 3.1 "Encoding" and section 3.3 "Per-row scale"):
// every weight x becomes the greedy 5-step ternary path c_1..c_5 over the
// ladder s_1..s_5 of r_0 = x / a, with a zero bias zeta that keeps c_i = 0
// while |r_{i-1}| < zeta s_i; a is the global alpha = max |W|, or the maximum
// |W| over the row's scale group (a row, or a head of rows_per_scale rows),
// whose rho = fp16(a / alpha) goes to the output.
//
// Three launches, HBM-bound, no memory beyond the outputs:
//   1. maxima: one warp per row reads the row once (16-byte loads), keeps its
//      largest bf16 magnitude, folds it into the group's maximum (held as a
//      bf16 bit pattern in rho_out, 16-bit atomic max) and the matrix maximum
//      (fp32 bits in alpha_out, 32-bit atomic max; magnitudes order like
//      their bit patterns). NaN / Inf weights are skipped and reported.
//   2. encode: each thread turns 8 weights (one 16-byte load) into 8 codes
//      (one 8-byte store).
//   3. rho: rho[g] = fp16(a_g / alpha) over the group maxima.
// The digit decisions use the arithmetic the oracle fixes: r_0 = fp32(x / a)
// (IEEE division), threshold fp32(zeta * s_i) (computed on the host), the
// non-zero candidate with the sign of r taken only when |fp32(r - c s_i)| <
// |r|, then r = fp32(r - c_i s_i); code = sum (c_i + 1) 3^(i-1).
#include "tq_common.cuh"

namespace tq {
namespace {

struct Ladder {
  float s[5];   // amplitudes s_1..s_5
  float zs[5];  // fp32(zeta * s_i)
};

__device__ __forceinline__ void atomic_max_u16(uint16_t *addr, uint16_t v) {
  unsigned short *a = reinterpret_cast<unsigned short *>(addr);
  unsigned short old = *reinterpret_cast<volatile unsigned short *>(a);
  while (old < v) {
    const unsigned short prev = atomicCAS(a, old, (unsigned short)v);
    if (prev == old) break;
    old = prev;
  }
}

// Largest finite bf16 magnitude of the 8 weights in w (as a bit pattern);
// sets *bad when one of them is NaN or Inf.
__device__ __forceinline__ uint32_t max_mag8(uint4 w, bool *bad) {
  const uint32_t v[4] = {w.x, w.y, w.z, w.w};
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t mag = (v[i] >> (16 * h)) & 0x7FFFu;
      if (mag >= 0x7F80u) {
        *bad = true;
      } else if (mag > m) {
        m = mag;
      }
    }
  }
  return m;
}

__global__ void encode_max_kernel(const uint4 *__restrict__ W, int64_t n,
                                  int64_t kc, int rps, uint16_t *group_max,
                                  uint32_t *alpha_bits, int32_t *status) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  uint32_t cta_max = 0;
  bool bad = false;
  for (int64_t row = warp0; row < n; row += warps) {
    const uint4 *p = W + row * kc;
    uint32_t m = 0;
    for (int64_t j = lane; j < kc; j += 32) {
      const uint32_t v = max_mag8(__ldg(p + j), &bad);
      m = v > m ? v : m;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const uint32_t t = __shfl_xor_sync(0xFFFFFFFFu, m, o);
      m = t > m ? t : m;
    }
    if (lane == 0 && rps > 0) atomic_max_u16(group_max + row / rps, (uint16_t)m);
    cta_max = m > cta_max ? m : cta_max;
  }
  // bf16 magnitude -> fp32 bit pattern keeps the order
  __shared__ uint32_t smax;
  if (threadIdx.x == 0) smax = 0;
  __syncthreads();
  atomicMax(&smax, cta_max << 16);
  if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) report(status, TQ_ERR_NONFINITE);
  __syncthreads();
  if (threadIdx.x == 0 && smax != 0) atomicMax(alpha_bits, smax);
}

__device__ __forceinline__ uint32_t encode_weight(float r, const Ladder &L) {
  uint32_t code = 0, p3 = 1;
#pragma unroll
  for (int i = 0; i < 5; ++i) {
    const float ar = fabsf(r);
    uint32_t d = 1;  // digit c_i + 1
    if (!(ar < L.zs[i]) && r != 0.0f) {
      const bool pos = r > 0.0f;
      const float rn = pos ? __fsub_rn(r, L.s[i]) : __fadd_rn(r, L.s[i]);
      if (fabsf(rn) < ar) {
        d = pos ? 2u : 0u;
        r = rn;
      }
    }
    code += d * p3;
    p3 *= 3u;
  }
  return code;
}

__global__ void encode_codes_kernel(const uint4 *__restrict__ W, int64_t n,
                                    int64_t kc, int rps,
                                    const uint16_t *__restrict__ group_max,
                                    const uint32_t *__restrict__ alpha_bits,
                                    const Ladder L, uint2 *__restrict__ codes) {
  const float alpha = __uint_as_float(*alpha_bits);
  const int64_t total = n * kc;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    float a = alpha;
    if (rps > 0) a = __uint_as_float((uint32_t)group_max[(i / kc) / rps] << 16);
    const uint4 w = __ldg(W + i);
    const uint32_t v[4] = {w.x, w.y, w.z, w.w};
    uint32_t out[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float x = __uint_as_float(((v[e >> 1] >> (16 * (e & 1))) & 0xFFFFu) << 16);
      const float r0 = a == 0.0f ? 0.0f : __fdiv_rn(x, a);
      out[e >> 2] |= encode_weight(r0, L) << (8 * (e & 3));
    }
    codes[i] = make_uint2(out[0], out[1]);
  }
}

__global__ void encode_rho_kernel(uint16_t *rho, int64_t groups,
                                  const uint32_t *__restrict__ alpha_bits) {
  const double alpha = (double)__uint_as_float(*alpha_bits);
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < groups;
       g += (int64_t)gridDim.x * blockDim.x) {
    const double a = (double)__uint_as_float((uint32_t)rho[g] << 16);
    rho[g] = a == 0.0 ? (uint16_t)0
                      : __half_as_ushort(__double2half(__ddiv_rn(a, alpha)));
  }
}

}  // namespace

cudaError_t launch_encode_b(const uint16_t *W, int64_t n, int64_t k,
                            const float ladder[5], float zeta, int rps,
                            uint8_t *codes, uint16_t *rho, float *alpha,
                            int32_t *status, cudaStream_t stream) {
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t groups = rps > 0 ? (n + rps - 1) / rps : 0;
  if ((e = cudaMemsetAsync(alpha, 0, sizeof(float), stream)) != cudaSuccess)
    return e;
  if (groups > 0 &&
      (e = cudaMemsetAsync(rho, 0, (size_t)groups * 2, stream)) != cudaSuccess)
    return e;
  if (n == 0 || k == 0) return cudaSuccess;
  const int64_t kc = k / 8;  // 16-byte chunks per row
  Ladder L;
  for (int i = 0; i < 5; ++i) {
    L.s[i] = ladder[i];
    L.zs[i] = zeta * ladder[i];  // one fp32 rounding
  }
  const uint4 *W4 = reinterpret_cast<const uint4 *>(W);
  uint32_t *abits = reinterpret_cast<uint32_t *>(alpha);
  {
    const int threads = 256;
    const int64_t want = (n + 7) / 8;  // 8 rows (warps) per CTA
    const int grid = (int)(want < 8LL * sms ? want : 8LL * sms);
    encode_max_kernel<<<grid, threads, 0, stream>>>(W4, n, kc, rps, rho,
                                                    abits, status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    const int threads = 256;
    const int64_t total = n * kc;
    const int64_t want = (total + threads - 1) / threads;
    const int grid = (int)(want < 16LL * sms ? want : 16LL * sms);
    encode_codes_kernel<<<grid, threads, 0, stream>>>(
        W4, n, kc, rps, rho, abits, L, reinterpret_cast<uint2 *>(codes));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (groups > 0) {
    const int threads = 256;
    const int64_t want = (groups + threads - 1) / threads;
    const int grid = (int)(want < 4LL * sms ? want : 4LL * sms);
    encode_rho_kernel<<<grid, threads, 0, stream>>>(rho, groups, abits);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace tq
