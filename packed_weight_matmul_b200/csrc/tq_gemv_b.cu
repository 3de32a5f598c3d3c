// Format B fused GEMV for small batches (alphaneural.io page, sections 3.2,
// 3.3 and 4.2): y[b][n] = rho[n / rps] * sum_k LUT[code[n][k]] * x[b][k].
//
// HBM-bound: one code byte per weight is read once; everything else lives on
// chip.
//   - Grid: one CTA per resident slot (a multiple of the SM count); CTA i
//     owns rows [i*n/P, (i+1)*n/P), an even share of the matrix.
//   - Inside a CTA every warp sees every row of the CTA but only its own
//     k-chunks (chunk = 32 lanes x KPL codes): the chunk count is chosen per
//     shape so that it divides evenly among the warps.
//   - x for the warp's chunk is converted once to fp32 and kept in registers
//     while the warp walks the CTA's rows, R rows at a time, with the next
//     group's code loads in flight (128-bit coalesced loads, streamed).
//   - The 243-entry code book is replicated once per lane in shared memory:
//     entry e of lane l's copy sits at byte e*256 + 4*l (all 256 byte
//     values, so an invalid code reads its NaN entry), so a warp's 32
//     random lookups hit 32 distinct banks, and one byte-permute builds the
//     address from the code byte.
//   - Products accumulate in fp32 with packed FFMA2 over k pairs; per row
//     group the R*B partial sums are reduced across lanes with a transposing
//     butterfly (about 2 shuffles per value instead of 5), summed over the
//     warp's chunks in shared memory, then over warps in a fixed order:
//     deterministic.
#include "tq_common.cuh"
#include "tq_linear.cuh"

namespace tq {
namespace {

constexpr int kLutStride = 256;                 // bytes per code-book entry
constexpr int kLutBytes = 256 * kLutStride;     // all byte values: 64 KB
constexpr int kMaxWarps = 8;
constexpr int kCtasPerSm = 2;

__device__ __forceinline__ uint4 ld_stream16(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint2 ld_stream8(const void *p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
               : "=r"(v.x), "=r"(v.y)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t ld_stream4(const void *p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];"
               : "=r"(v)
               : "l"(p));
  return v;
}

// Load KPL code bytes as KPL/4 words.
template <int KPL>
__device__ __forceinline__ void load_codes(const uint8_t *p, uint32_t *w) {
  if constexpr (KPL == 16) {
    const uint4 v = ld_stream16(p);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (KPL == 8) {
    const uint2 v = ld_stream8(p);
    w[0] = v.x; w[1] = v.y;
  } else {
    w[0] = ld_stream4(p);
  }
}

// bf16 pair (low half = lower k) -> float2.
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

// Code-book value of byte q of word w for this lane (lane4 = 4 * lane).
__device__ __forceinline__ float lut_at(const uint8_t *lut_smem, uint32_t w,
                                        int q, uint32_t lane4) {
  // result bytes: [0] = lane4, [1] = code byte q, [2], [3] = 0 (lane4 < 256)
  const uint32_t addr = __byte_perm(w, lane4, 0x5504u | ((uint32_t)q << 4));
  return *reinterpret_cast<const float *>(lut_smem + addr);
}

// Reduce M (power of two, <= 32) per-lane values across the warp. On return
// lane l holds, in v[0], the full sum of value index l >> (5 - log2 M).
template <int M>
__device__ __forceinline__ float butterfly_reduce(float *v, int lane) {
  int m = M;
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    if (m > 1) {
      const int h = m / 2;
      const bool upper = (lane & s) != 0;
#pragma unroll
      for (int i = 0; i < h; ++i) {
        const float send = upper ? v[i] : v[i + h];
        const float keep = upper ? v[i + h] : v[i];
        v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, s);
      }
      m = h;
    } else {
      v[0] += __shfl_xor_sync(0xFFFFFFFFu, v[0], s);
    }
  }
  return v[0];
}

template <int B>
struct RowsPerGroup {
  static constexpr int value = (B <= 2) ? 4 : ((B <= 4) ? 4 : 2);
};

constexpr int pow2_ceil(int v) {
  int p = 1;
  while (p < v) p *= 2;
  return p;
}

template <int B, int KPL>
__global__ void __launch_bounds__(kMaxWarps * 32, kCtasPerSm)
    gemv_b_kernel(const uint8_t *__restrict__ codes, int64_t n, int64_t k,
                  const float *__restrict__ lut,
                  const uint16_t *__restrict__ rho, int rps,
                  const __nv_bfloat16 *__restrict__ x, int64_t ldx,
                  float *__restrict__ y, int64_t ldy, int rows_max) {
  constexpr int R = RowsPerGroup<B>::value;
  constexpr int M = pow2_ceil(R * B);  // values reduced per row group
  constexpr int KC = 32 * KPL;         // k per warp chunk
  constexpr int NW = KPL / 4;          // code words per lane per row
  extern __shared__ __align__(16) uint8_t smem[];
  float *red = reinterpret_cast<float *>(smem + kLutBytes);  // [warps][rows_max][B]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int64_t row_lo = (int64_t)blockIdx.x * n / gridDim.x;
  const int rows = (int)((int64_t)(blockIdx.x + 1) * n / gridDim.x - row_lo);
  const uint8_t *crow = codes + row_lo * k;

  // Replicate the code book (all 256 entries, so an invalid code reads its
  // NaN entry): word e*64 + l holds LUT[e] for lane l.
  float *lut_words = reinterpret_cast<float *>(smem);
  for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x)
    lut_words[(i >> 5) * 64 + (i & 31)] = __ldg(lut + (i >> 5));
  for (int i = threadIdx.x; i < nwarps * rows_max * B; i += blockDim.x)
    red[i] = 0.0f;
  __syncthreads();

  const uint32_t lane4 = (uint32_t)lane * 4u;
  const int64_t nchunks = (k + KC - 1) / KC;
  for (int64_t c = warp; c < nchunks; c += nwarps) {
    const int64_t kb = c * KC + (int64_t)lane * KPL;
    const bool valid = kb < k;  // k % 16 == 0: a lane is all in or all out
    float2 xv[B][KPL / 2];
#pragma unroll
    for (int b = 0; b < B; ++b) {
      if (valid) {
        const __nv_bfloat16 *xp = x + b * ldx + kb;
        uint32_t u[KPL / 2];
        if constexpr (KPL == 16) {
          const uint4 a = *reinterpret_cast<const uint4 *>(xp);
          const uint4 d = *reinterpret_cast<const uint4 *>(xp + 8);
          u[0] = a.x; u[1] = a.y; u[2] = a.z; u[3] = a.w;
          u[4] = d.x; u[5] = d.y; u[6] = d.z; u[7] = d.w;
        } else if constexpr (KPL == 8) {
          const uint4 a = *reinterpret_cast<const uint4 *>(xp);
          u[0] = a.x; u[1] = a.y; u[2] = a.z; u[3] = a.w;
        } else {
          const uint2 a = *reinterpret_cast<const uint2 *>(xp);
          u[0] = a.x; u[1] = a.y;
        }
#pragma unroll
        for (int i = 0; i < KPL / 2; ++i) xv[b][i] = bf16x2_to_float2(u[i]);
      } else {
#pragma unroll
        for (int i = 0; i < KPL / 2; ++i) xv[b][i] = make_float2(0.f, 0.f);
      }
    }

    // software pipeline over row groups: codes of group g+1 load during g
    uint32_t cw[R][NW], cn[R][NW];
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
      for (int i = 0; i < NW; ++i) cw[r][i] = 0x79797979u;  // code 121 = 0
      if (valid && r < rows) load_codes<KPL>(crow + (int64_t)r * k + kb, cw[r]);
    }
    for (int r0 = 0; r0 < rows; r0 += R) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
#pragma unroll
        for (int i = 0; i < NW; ++i) cn[r][i] = 0x79797979u;
        const int rn = r0 + R + r;
        if (valid && rn < rows)
          load_codes<KPL>(crow + (int64_t)rn * k + kb, cn[r]);
      }
      float2 acc[R][B];
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int b = 0; b < B; ++b) acc[r][b] = make_float2(0.f, 0.f);
#pragma unroll
      for (int r = 0; r < R; ++r) {
#pragma unroll
        for (int i = 0; i < NW; ++i) {
#pragma unroll
          for (int q = 0; q < 4; q += 2) {
            const float2 wv = make_float2(lut_at(smem, cw[r][i], q, lane4),
                                          lut_at(smem, cw[r][i], q + 1, lane4));
#pragma unroll
            for (int b = 0; b < B; ++b)
              acc[r][b] = __ffma2_rn(wv, xv[b][i * 2 + q / 2], acc[r][b]);
          }
        }
      }
      float v[M];
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int b = 0; b < B; ++b) v[r * B + b] = acc[r][b].x + acc[r][b].y;
#pragma unroll
      for (int i = R * B; i < M; ++i) v[i] = 0.0f;
      const float s = butterfly_reduce<M>(v, lane);
      constexpr int kLowBits = 32 / M;  // lanes sharing one reduced value
      const int idx = lane / kLowBits;
      if ((lane % kLowBits) == 0 && idx < R * B) {
        const int r = idx / B, b = idx % B;
        if (r0 + r < rows) red[(warp * rows_max + r0 + r) * B + b] += s;
      }
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int i = 0; i < NW; ++i) cw[r][i] = cn[r][i];
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < rows * B; i += blockDim.x) {
    const int r = i / B, b = i % B;
    float s = 0.0f;
    for (int w = 0; w < nwarps; ++w) s += red[(w * rows_max + r) * B + b];
    const int64_t row = row_lo + r;
    const float scale =
        rho ? __half2float(__ushort_as_half(rho[row / rps])) : 1.0f;
    y[(int64_t)b * ldy + row] = scale * s;
  }
}

// Pick the lane width KPL (codes per lane per chunk) and the warp count so
// that the k-chunks divide evenly among the warps of a CTA.
struct ChunkPlan {
  int kpl;
  int warps;
};

ChunkPlan plan_chunks(int64_t k, int kpl_max) {
  ChunkPlan best{4, 1};
  double best_eff = -1.0;
  for (int kpl = kpl_max; kpl >= 4; kpl /= 2) {
    const int64_t nchunks = (k + 32 * kpl - 1) / (32 * kpl);
    const int wmax = (int)(nchunks < kMaxWarps ? nchunks : kMaxWarps);
    for (int w = wmax; w >= 1 && w >= wmax - 4; --w) {
      const int64_t rounds = (nchunks + w - 1) / w;
      // useful lane-chunks over issued lane-chunks (a partial last chunk
      // counts by its valid lanes)
      const double useful = (double)k / (32.0 * kpl);
      const double eff = useful / (double)(rounds * w) * (w >= 4 ? 1.0 : 0.9);
      if (eff > best_eff + 1e-9) {
        best_eff = eff;
        best = ChunkPlan{kpl, w};
      }
    }
  }
  return best;
}

template <int B, int KPL>
cudaError_t launch_kpl(const WeightsView &w, const __nv_bfloat16 *x,
                       int64_t ldx, float *y, int64_t ldy, int warps,
                       cudaStream_t stream) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  constexpr int kMaxRedBytes = 96 * 1024;
  const int64_t rows_cap = kMaxRedBytes / (warps * B * 4);
  int64_t ctas = (int64_t)sms * kCtasPerSm;
  if ((w.n + ctas - 1) / ctas > rows_cap) ctas = (w.n + rows_cap - 1) / rows_cap;
  if (ctas > w.n) ctas = w.n;
  const int rows_max = (int)((w.n + ctas - 1) / ctas);
  const size_t smem = kLutBytes + (size_t)warps * rows_max * B * sizeof(float);
  auto kern = gemv_b_kernel<B, KPL>;
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)ctas, warps * 32, smem, stream>>>(
      w.codes, w.n, w.k, w.lut, w.scales, w.rps, x, ldx, y, ldy, rows_max);
  return cudaGetLastError();
}

template <int B>
cudaError_t launch_b(const WeightsView &w, const __nv_bfloat16 *x, int64_t ldx,
                     float *y, int64_t ldy, cudaStream_t stream) {
  constexpr int kplMax = (B <= 2) ? 16 : ((B <= 4) ? 8 : 4);
  const ChunkPlan p = plan_chunks(w.k, kplMax);
  if (p.kpl == 16) {
    if constexpr (kplMax >= 16)
      return launch_kpl<B, 16>(w, x, ldx, y, ldy, p.warps, stream);
  }
  if (p.kpl >= 8) {
    if constexpr (kplMax >= 8)
      return launch_kpl<B, 8>(w, x, ldx, y, ldy, p.warps, stream);
  }
  return launch_kpl<B, 4>(w, x, ldx, y, ldy, p.warps, stream);
}

}  // namespace

bool gemv_b_supported(const WeightsView &w, int64_t batch) {
  return w.format == TQ_FMT_B && batch >= 1 && batch <= 8;
}

cudaError_t gemv_b(const WeightsView &w, const __nv_bfloat16 *x, int64_t batch,
                   int64_t ldx, float *y, int64_t ldy, cudaStream_t stream) {
  switch (batch) {
    case 1: return launch_b<1>(w, x, ldx, y, ldy, stream);
    case 2: return launch_b<2>(w, x, ldx, y, ldy, stream);
    case 3: return launch_b<3>(w, x, ldx, y, ldy, stream);
    case 4: return launch_b<4>(w, x, ldx, y, ldy, stream);
    case 5: return launch_b<5>(w, x, ldx, y, ldy, stream);
    case 6: return launch_b<6>(w, x, ldx, y, ldy, stream);
    case 7: return launch_b<7>(w, x, ldx, y, ldy, stream);
    default: return launch_b<8>(w, x, ldx, y, ldy, stream);
  }
}

}  // namespace tq
