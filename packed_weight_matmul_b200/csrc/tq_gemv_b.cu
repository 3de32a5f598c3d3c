// Format B fused GEMV for small batches (alphaneural.io page, sections 3.2,
// 3.3 and 4.2): y[b][n] = rho[n / rps] * sum_k LUT[code[n][k]] * x[b][k].
//
// HBM-bound: one code byte per weight is read once; everything else lives on
// chip. The design keeps the per-weight instruction count near three (one
// byte permute, one shared load, one FFMA) and the SM full of warps:
//   - Grid: one CTA per SM; CTA i owns rows [i*n/P, (i+1)*n/P), an even share
//     of the matrix. The CTA is large (up to 32 warps) so that many 16-byte
//     code loads are in flight per SM while registers stay under 64.
//   - Warps are arranged as WK x WR: the WK warps of a row slice split the
//     k-chunks (chunk = 32 lanes x KPL codes; KPL and WK are chosen per shape
//     so the chunks divide evenly), the WR slices split the CTA's rows.
//   - x for the warp's chunk is converted to fp32 once and kept in registers
//     while the warp walks its rows, R at a time; the next row group's codes
//     (and, at a chunk's start, the next chunk's x) are loaded a step ahead,
//     128-bit, streaming past L1.
//   - The code book is replicated once per lane in shared memory: entry e of
//     lane l's copy sits at byte e*256 + 4*l, so a warp's 32 random lookups
//     hit 32 distinct banks, and one byte permute of the code word with 4*l
//     is the whole address. All 256 byte values are present, so an invalid
//     code reads its NaN entry.
//   - Per row group the R*B partial sums are reduced across lanes with a
//     transposing butterfly (about 2 shuffles per value instead of 5), summed
//     over the warp's chunks in shared memory and finally over the WK warps in
//     a fixed order: deterministic.
#include "tq_common.cuh"
#include "tq_linear.cuh"

namespace tq {
namespace {

constexpr int kLutStride = 256;              // bytes per code-book entry
constexpr int kLutBytes = 256 * kLutStride;  // all byte values: 64 KB

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

// bf16 pair (low half = lower k) -> float2.
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

// Code-book value of byte q of word w for this lane: the byte permute
// yields code*256 + 4*lane, added to the table's 32-bit shared address.
__device__ __forceinline__ float lut_at(uint32_t lut_base, uint32_t w, int q,
                                        uint32_t lane4) {
  const uint32_t a = __byte_perm(w, lane4, 0x5504u | ((uint32_t)q << 4));
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(lut_base + a));
  return v;
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

constexpr int pow2_ceil(int v) {
  int p = 1;
  while (p < v) p *= 2;
  return p;
}

template <int B>
struct GemvBCfg {
  static constexpr int R = (B <= 2) ? 4 : 2;          // rows per group
  static constexpr int kMaxThreads = (B == 1) ? 768 : 512;
};


template <int B, int KPL>
__global__ void __launch_bounds__(GemvBCfg<B>::kMaxThreads, 1)
    gemv_b_kernel(const uint8_t *__restrict__ codes, int64_t n, int64_t k,
                  const float *__restrict__ lut,
                  const uint16_t *__restrict__ rho, int rps,
                  const __nv_bfloat16 *__restrict__ x, int64_t ldx,
                  float *__restrict__ y, int64_t ldy, int wk_count,
                  int rows_max) {
  constexpr int R = GemvBCfg<B>::R;
  constexpr int M = pow2_ceil(R * B);  // values reduced per row group
  constexpr int KC = 32 * KPL;         // k per warp chunk
  constexpr int NW = KPL / 4;          // code words per lane per row
  extern __shared__ __align__(16) uint8_t smem[];
  float *red = reinterpret_cast<float *>(smem + kLutBytes);  // [WK][rows][B]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int wk = warp % wk_count, wr = warp / wk_count;
  const int wr_count = nwarps / wk_count;
  const int64_t row_lo = (int64_t)blockIdx.x * n / gridDim.x;
  const int rows = (int)((int64_t)(blockIdx.x + 1) * n / gridDim.x - row_lo);
  const int r_begin = rows * wr / wr_count;
  const int my_rows = rows * (wr + 1) / wr_count - r_begin;
  const uint8_t *crow = codes + (row_lo + r_begin) * k;
  const uint32_t kstride = (uint32_t)k;  // row pitch (k < 2^32)
  const int64_t nchunks = (k + KC - 1) / KC;
  const int nc_w = (int)((nchunks - wk + wk_count - 1) / wk_count);
  const int ng = (my_rows + R - 1) / R;
  const int total = nc_w * ng;

  auto kb_of = [&](int ci) -> int64_t {
    return (wk + (int64_t)ci * wk_count) * KC + (int64_t)lane * KPL;
  };
  // Codes of chunk ci, row group g; 121 (weight 0) where there is nothing to
  // load. (No integer division in the loop: divisions run on the slow
  // conversion pipe.)
  auto load_group = [&](int ci, int g, uint32_t (&cw)[R][NW]) {
    const int64_t kb = kb_of(ci);
    const bool ok_i = ci < nc_w && kb < k;
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
      for (int q = 0; q < NW; ++q) cw[r][q] = 0x79797979u;
      const int row = g * R + r;
      if (ok_i && row < my_rows) {
        const uint8_t *p = crow + (int64_t)row * kstride + kb;
        if constexpr (KPL == 16) {
          const uint4 v = ld_stream16(p);
          cw[r][0] = v.x; cw[r][1] = v.y; cw[r][2] = v.z; cw[r][3] = v.w;
        } else {
          const uint2 v = ld_stream8(p);
          cw[r][0] = v.x; cw[r][1] = v.y;
        }
      }
    }
  };
  // Raw bf16 words of x for chunk ci (this lane's KPL columns).
  uint32_t xr[B][KPL / 2];
  auto load_x = [&](int ci) {
    const int64_t kb = kb_of(ci);
    const bool ok = ci < nc_w && kb < k;
#pragma unroll
    for (int b = 0; b < B; ++b) {
#pragma unroll
      for (int q = 0; q < KPL / 2; q += 4) {
        uint4 v = make_uint4(0, 0, 0, 0);
        if (ok) v = *reinterpret_cast<const uint4 *>(x + b * ldx + kb + 2 * q);
        xr[b][q] = v.x;
        xr[b][q + 1] = v.y;
        xr[b][q + 2] = v.z;
        xr[b][q + 3] = v.w;
      }
    }
  };

  // Start the first loads, then build the code book while they fly.
  uint32_t cw[R][NW], cn[R][NW];
  load_group(0, 0, cw);
  load_x(0);
  // Replicate the code book, coalesced loads and conflict-free 16 B stores:
  // entry e's 32 lane copies are 8 float4 chunks, written in rotated order.
  for (int e = threadIdx.x; e < 256; e += blockDim.x) {
    const float v = __ldg(lut + e);
    const float4 v4 = make_float4(v, v, v, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int jj = (j + e) & 7;
      *reinterpret_cast<float4 *>(smem + e * kLutStride + jj * 16) = v4;
    }
  }
  for (int i = threadIdx.x; i < wk_count * rows_max * B; i += blockDim.x)
    red[i] = 0.0f;
  __syncthreads();

  const uint32_t lane4 = (uint32_t)lane * 4u;
  const uint32_t lut_base = (uint32_t)__cvta_generic_to_shared(smem);
  float xv[B][KPL];
  bool lane_ok = false;
  int ci = 0, g = 0;  // current chunk and row group
  for (int i = 0; i < total; ++i) {
    const bool wrap = g + 1 == ng;
    load_group(wrap ? ci + 1 : ci, wrap ? 0 : g + 1, cn);  // one group ahead
    if (g == 0) {
      lane_ok = kb_of(ci) < k;
#pragma unroll
      for (int b = 0; b < B; ++b)
#pragma unroll
        for (int q = 0; q < KPL / 2; ++q) {
          xv[b][2 * q] = __uint_as_float(xr[b][q] << 16);
          xv[b][2 * q + 1] = __uint_as_float(xr[b][q] & 0xFFFF0000u);
        }
      load_x(ci + 1);  // next chunk's x, consumed ng groups later
    }
    float acc[R][B];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int b = 0; b < B; ++b) acc[r][b] = 0.0f;
    if (lane_ok) {
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int q = 0; q < NW; ++q)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float wv = lut_at(lut_base, cw[r][q], e, lane4);
#pragma unroll
            for (int b = 0; b < B; ++b)
              acc[r][b] = fmaf(wv, xv[b][q * 4 + e], acc[r][b]);
          }
    }
    float v[M];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int b = 0; b < B; ++b) v[r * B + b] = acc[r][b];
#pragma unroll
    for (int q = R * B; q < M; ++q) v[q] = 0.0f;
    const float s = butterfly_reduce<M>(v, lane);
    constexpr int kLow = 32 / M;  // lanes holding the same reduced value
    const int idx = lane / kLow;
    if ((lane % kLow) == 0 && idx < R * B) {
      const int r = idx / B, b = idx % B;
      const int row = g * R + r;
      if (row < my_rows)
        red[(wk * rows_max + r_begin + row) * B + b] += s;
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int q = 0; q < NW; ++q) cw[r][q] = cn[r][q];
    if (wrap) {
      ++ci;
      g = 0;
    } else {
      ++g;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < rows * B; i += blockDim.x) {
    const int r = i / B, b = i % B;
    float s = 0.0f;
    for (int w = 0; w < wk_count; ++w) s += red[(w * rows_max + r) * B + b];
    const int64_t row = row_lo + r;
    const float scale =
        rho ? __half2float(__ushort_as_half(rho[row / rps])) : 1.0f;
    y[(int64_t)b * ldy + row] = scale * s;
  }
}

// Warp layout and lane width for one shape: the k-chunks split evenly over
// WK warps, WR row slices fill the CTA.
struct GemvPlan {
  int kpl;
  int wk;
  int wr;
};

GemvPlan plan_gemv(int64_t k, int64_t rows_per_cta, int max_warps, int R,
                   int kpl_max) {
  GemvPlan best{8, 1, 1};
  double best_score = -1.0;
  for (int kpl = kpl_max; kpl >= 8; kpl /= 2) {
    const int64_t nchunks = (k + 32 * kpl - 1) / (32 * kpl);
    const double useful = (double)k / (32.0 * kpl);
    for (int wk = 1; wk <= max_warps && wk <= nchunks; ++wk) {
      const int64_t rounds = (nchunks + wk - 1) / wk;
      const double eff = useful / (double)(rounds * wk);
      int wr = max_warps / wk;
      const int64_t wr_rows = (rows_per_cta + R - 1) / R;  // >= R rows each
      if (wr > wr_rows) wr = (int)(wr_rows > 0 ? wr_rows : 1);
      const double score = eff * (double)(wk * wr) / max_warps;
      if (score > best_score + 1e-9) {
        best_score = score;
        best = GemvPlan{kpl, wk, wr};
      }
    }
  }
  return best;
}

template <int B, int KPL>
cudaError_t launch_kpl(const WeightsView &w, const __nv_bfloat16 *x,
                       int64_t ldx, float *y, int64_t ldy, int64_t ctas,
                       const GemvPlan &p, cudaStream_t stream) {
  const int rows_max = (int)((w.n + ctas - 1) / ctas);
  const size_t smem =
      kLutBytes + (size_t)p.wk * rows_max * B * sizeof(float);
  auto kern = gemv_b_kernel<B, KPL>;
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)ctas, p.wk * p.wr * 32, smem, stream>>>(
      w.codes, w.n, w.k, w.lut, w.scales, w.rps, x, ldx, y, ldy, p.wk,
      rows_max);
  return cudaGetLastError();
}

template <int B>
cudaError_t launch_b(const WeightsView &w, const __nv_bfloat16 *x, int64_t ldx,
                     float *y, int64_t ldy, cudaStream_t stream) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  constexpr int kMaxWarps = GemvBCfg<B>::kMaxThreads / 32;
  int64_t ctas = sms;
  // keep the partial-sum buffer small (<= 96 KB): more CTAs for tall shapes
  const int64_t rows_cap = (96 * 1024) / (kMaxWarps * B * 4);
  if ((w.n + ctas - 1) / ctas > rows_cap) ctas = (w.n + rows_cap - 1) / rows_cap;
  if (ctas > w.n) ctas = w.n;
  constexpr int kKplMax = (B <= 2) ? 16 : 8;  // register budget
  const GemvPlan p = plan_gemv(w.k, (w.n + ctas - 1) / ctas, kMaxWarps,
                               GemvBCfg<B>::R, kKplMax);
  if constexpr (kKplMax == 16) {
    if (p.kpl == 16)
      return launch_kpl<B, 16>(w, x, ldx, y, ldy, ctas, p, stream);
  }
  return launch_kpl<B, 8>(w, x, ldx, y, ldy, ctas, p, stream);
}

}  // namespace

bool gemv_b_supported(const WeightsView &w, int64_t batch) {
  return w.format == TQ_FMT_B && batch >= 1 && batch <= 4;
}

cudaError_t gemv_b(const WeightsView &w, const __nv_bfloat16 *x, int64_t batch,
                   int64_t ldx, float *y, int64_t ldy, cudaStream_t stream) {
  switch (batch) {
    case 1: return launch_b<1>(w, x, ldx, y, ldy, stream);
    case 2: return launch_b<2>(w, x, ldx, y, ldy, stream);
    case 3: return launch_b<3>(w, x, ldx, y, ldy, stream);
    default: return launch_b<4>(w, x, ldx, y, ldy, stream);
  }
}

}  // namespace tq
