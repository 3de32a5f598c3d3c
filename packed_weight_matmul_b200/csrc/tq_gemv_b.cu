// Format B fused GEMV for small batches (alphaneural.io page, sections 3.2,
// 3.3 and 4.2): y[b][n] = rho[n / rps] * sum_k LUT[code[n][k]] * x[b][k].
//
// HBM-bound: one code byte per weight is read once; everything else lives on
// chip. At full bandwidth an SM must retire 22 weights per clock, which
// leaves about five warp instructions per 32 weights, so the inner loop is
// two byte permutes, two shared loads and B packed FMAs per weight pair:
//   - The code book is replicated once per lane at shared-window address
//     64 KB: entry e of lane l's copy is at 0x10000 + e*256 + 4*l. A byte
//     permute of the code word with (0x10000 | 4*l) is then the complete
//     address, a warp's 32 lookups hit 32 distinct banks, and all 256 byte
//     values are present, so an invalid code reads its NaN entry.
//   - Two neighbouring weights are multiplied by their two x values with one
//     packed fp32x2 FMA (even and odd k accumulate separately and are added
//     at the end of a unit).
//   - Work unit: R rows x one k-chunk of 32 lanes x KPL codes (16-byte or
//     8-byte loads per lane and row, a fully coalesced 512- or 256-byte run
//     per row). A CTA (one per SM) owns an even share of the rows; its units
//     are ordered chunk-major and cut into equal contiguous ranges, one per
//     warp, so every warp does the same amount of work (+-1 unit) and keeps
//     the chunk's x in registers across the row groups it walks.
//   - Codes of the next D-1 units are in flight while a unit is computed (a
//     register ring, 128-bit loads that bypass L1); the x of the next chunk
//     is fetched while the current chunk is in use.
//   - A unit's R*B sums are reduced across lanes by a transposing butterfly
//     and written to a per-(chunk, row) slot in shared memory; the slots of a
//     row are added in chunk order at the end, so the result does not depend
//     on timing.
#include "tq_common.cuh"
#include "tq_linear.cuh"

namespace tq {
namespace {

constexpr uint32_t kLutAddr = 0x10000u;  // shared-window address of the book
constexpr uint32_t kLutStride = 256;     // bytes per entry (32 lane copies)
constexpr uint32_t kRedAddr = 0x20000u;  // partial sums follow the book
constexpr int kSmemMax = 227 * 1024;     // dynamic shared memory per CTA
// The request covers [0, kRedAddr + red) whatever the window base is.
constexpr int kRedMaxBytes = kSmemMax - (int)kRedAddr;

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

__device__ __forceinline__ float lds_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}

__device__ __forceinline__ void sts_f32(uint32_t a, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}

__device__ __forceinline__ void sts_v4(uint32_t a, float v) {
  asm volatile("st.shared.v4.f32 [%0], {%1,%1,%1,%1};" ::"r"(a), "f"(v)
               : "memory");
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

// Position of a work unit: chunk c, row group g, and the byte offset of this
// lane's codes for the group's first row.
struct UnitPos {
  int c, g;
  int64_t off;
};

template <int B, int KPL, int R, int D, int NT>
__global__ void __launch_bounds__(NT, 1)
    gemv_b_kernel(const uint8_t *__restrict__ codes, int64_t n, int64_t k,
                  const float *__restrict__ lut,
                  const uint16_t *__restrict__ rho, int rps,
                  const __nv_bfloat16 *__restrict__ x, int64_t ldx,
                  float *__restrict__ y, int64_t ldy, int rows_max) {
  constexpr int KC = 32 * KPL;         // k per chunk
  constexpr int NW = KPL / 4;          // code words per lane and row
  constexpr int NX = KPL / 2;          // x pairs per lane and batch row
  constexpr int M = pow2_ceil(R * B);  // values reduced per unit
  constexpr int kWarps = NT / 32;
  extern __shared__ __align__(16) uint8_t smem[];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row_lo = (int64_t)blockIdx.x * n / gridDim.x;
  const int rows = (int)((int64_t)(blockIdx.x + 1) * n / gridDim.x - row_lo);

  // The code book must start exactly at kLutAddr; the request size makes the
  // window reach kRedAddr + partial sums when the base is at most kLutAddr.
  const uint32_t base = (uint32_t)__cvta_generic_to_shared(smem);
  if (base > kLutAddr) {
    for (int i = threadIdx.x; i < rows * B; i += NT) {
      const int r = i / B, b = i - r * B;
      y[(int64_t)b * ldy + row_lo + r] = __int_as_float(0x7FC00000);
    }
    return;
  }

  const int ng = (rows + R - 1) / R;
  const int nchunks = (int)((k + KC - 1) / KC);
  const int units = ng * nchunks;
  const int u_begin = (int)((int64_t)units * warp / kWarps);
  const int u_end = (int)((int64_t)units * (warp + 1) / kWarps);
  const int64_t kstride = k;
  const int64_t group_step = (int64_t)R * kstride;
  const uint8_t *crow = codes + row_lo * kstride + lane * KPL;

  UnitPos ld;  // next unit whose codes are loaded
  ld.c = u_begin / ng;
  ld.g = u_begin - ld.c * ng;
  ld.off = (int64_t)ld.g * group_step + (int64_t)ld.c * KC;
  int u_ld = u_begin;
  UnitPos cur = ld;

  auto advance = [&](UnitPos &p) {
    if (++p.g == ng) {
      p.g = 0;
      ++p.c;
      p.off = (int64_t)p.c * KC;
    } else {
      p.off += group_step;
    }
  };
  auto lane_in_k = [&](int c) { return (int64_t)c * KC + lane * KPL < k; };

  // Codes of unit u_ld into slot cw, 121 (weight 0) where nothing is loaded.
  auto issue = [&](uint32_t (&cw)[R][NW]) {
    const bool ok = u_ld < u_end && lane_in_k(ld.c);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const bool okr = ok && ld.g * R + r < rows;
      const uint8_t *p = crow + ld.off + r * kstride;
      if constexpr (KPL == 16) {
        uint4 v = make_uint4(0x79797979u, 0x79797979u, 0x79797979u,
                             0x79797979u);
        if (okr) v = ld_stream16(p);
        cw[r][0] = v.x; cw[r][1] = v.y; cw[r][2] = v.z; cw[r][3] = v.w;
      } else {
        uint2 v = make_uint2(0x79797979u, 0x79797979u);
        if (okr) v = ld_stream8(p);
        cw[r][0] = v.x; cw[r][1] = v.y;
      }
    }
    if (u_ld < u_end) advance(ld);
    ++u_ld;
  };

  // Raw bf16 x words of chunk c for this lane (zero outside k).
  uint32_t xr[B][NX];
  auto load_x = [&](int c) {
    const bool ok = c < nchunks && lane_in_k(c);
    const int64_t kb = (int64_t)c * KC + lane * KPL;
#pragma unroll
    for (int b = 0; b < B; ++b) {
#pragma unroll
      for (int q = 0; q < NX; q += 4) {
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
  uint32_t cw[D][R][NW];
#pragma unroll
  for (int d = 0; d < D; ++d) issue(cw[d]);
  load_x(cur.c);
  for (int i = threadIdx.x; i < 256 * 8; i += NT) {
    const int e = i >> 3, j = i & 7;
    sts_v4(kLutAddr + e * kLutStride + j * 16, __ldg(lut + e));
  }
  __syncthreads();

  const uint32_t lane_lut = kLutAddr | ((uint32_t)lane << 2);
  float2 xv[B][NX];
  int xc = -1;  // chunk whose x is in xv
  bool k_ok = false;

  auto process = [&](const uint32_t (&cw)[R][NW]) {
    if (cur.c != xc) {  // entering a new chunk: take its x, fetch the next
      xc = cur.c;
      k_ok = lane_in_k(xc);
#pragma unroll
      for (int b = 0; b < B; ++b)
#pragma unroll
        for (int q = 0; q < NX; ++q)
          xv[b][q] = make_float2(__uint_as_float(xr[b][q] << 16),
                                 __uint_as_float(xr[b][q] & 0xFFFF0000u));
      load_x(xc + 1);
    }
    float2 acc[R][B];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int b = 0; b < B; ++b) acc[r][b] = make_float2(0.0f, 0.0f);
    if (k_ok) {
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int q = 0; q < NW; ++q)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t a0 =
                __byte_perm(cw[r][q], lane_lut, 0x7604u | ((2u * h) << 4));
            const uint32_t a1 =
                __byte_perm(cw[r][q], lane_lut, 0x7604u | ((2u * h + 1) << 4));
            const float2 wv = make_float2(lds_f32(a0), lds_f32(a1));
#pragma unroll
            for (int b = 0; b < B; ++b)
              acc[r][b] = __ffma2_rn(wv, xv[b][2 * q + h], acc[r][b]);
          }
    }
    float v[M];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int b = 0; b < B; ++b) v[r * B + b] = acc[r][b].x + acc[r][b].y;
#pragma unroll
    for (int q = R * B; q < M; ++q) v[q] = 0.0f;
    const float s = butterfly_reduce<M>(v, lane);
    constexpr int kLow = 32 / M;  // lanes holding the same reduced value
    const int idx = lane / kLow;
    if ((lane % kLow) == 0 && idx < R * B) {
      const int r = idx / B, b = idx - (idx / B) * B;
      const int row = cur.g * R + r;
      if (row < rows)
        sts_f32(kRedAddr + (uint32_t)(((cur.c * rows_max + row) * B + b) * 4),
                s);
    }
    advance(cur);
  };

  for (int u = u_begin; u < u_end; u += D) {
#pragma unroll
    for (int d = 0; d < D; ++d) {
      if (u + d < u_end) {
        process(cw[d]);
        issue(cw[d]);  // unit u + d + D
      }
    }
  }
  __syncthreads();

  for (int i = threadIdx.x; i < rows * B; i += NT) {
    const int r = i / B, b = i - r * B;
    float s = 0.0f;
    for (int c = 0; c < nchunks; ++c)
      s += lds_f32(kRedAddr + (uint32_t)(((c * rows_max + r) * B + b) * 4));
    const int64_t row = row_lo + r;
    const float scale =
        rho ? __half2float(__ushort_as_half(rho[row / rps])) : 1.0f;
    y[(int64_t)b * ldy + row] = scale * s;
  }
}

// Tile parameters of one launch.
struct GemvCfg {
  int kpl, r, d, nt;
};

template <int B, int KPL, int R, int D, int NT>
cudaError_t launch_cfg(const WeightsView &w, const __nv_bfloat16 *x,
                       int64_t ldx, float *y, int64_t ldy, int sms,
                       cudaStream_t stream) {
  constexpr int KC = 32 * KPL;
  const int64_t nchunks = (w.k + KC - 1) / KC;
  int64_t ctas = sms < w.n ? sms : w.n;
  // the partial sums (one slot per chunk, row and batch row) must fit
  const int64_t rows_cap = kRedMaxBytes / (nchunks * B * 4);
  if (rows_cap < 1) return cudaErrorInvalidValue;
  if ((w.n + ctas - 1) / ctas > rows_cap) ctas = (w.n + rows_cap - 1) / rows_cap;
  const int rows_max = (int)((w.n + ctas - 1) / ctas);
  const size_t smem = kRedAddr + (size_t)nchunks * rows_max * B * 4;
  auto kern = gemv_b_kernel<B, KPL, R, D, NT>;
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)ctas, NT, smem, stream>>>(w.codes, w.n, w.k, w.lut,
                                              w.scales, w.rps, x, ldx, y, ldy,
                                              rows_max);
  return cudaGetLastError();
}

int device_sms() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

// Row-group height for a shape: the largest R whose units still split
// evenly over the warps (at most ~12 % lost to the last partial unit).
int pick_rows(int64_t n, int64_t k, int kpl, int warps, int sms) {
  const int64_t nchunks = (k + 32 * kpl - 1) / (32 * kpl);
  const int64_t rows = (n + sms - 1) / sms;
  for (int r = 4; r >= 2; r /= 2) {
    const int64_t units = (rows + r - 1) / r * nchunks;
    const int64_t per_warp = (units + warps - 1) / warps;
    const double eff = (double)rows * nchunks / ((double)per_warp * warps * r);
    if (eff >= 0.88) return r;
  }
  return 2;
}

}  // namespace

bool gemv_b_supported(const WeightsView &w, int64_t batch) {
  return w.format == TQ_FMT_B && batch >= 1 && batch <= 4;
}

cudaError_t gemv_b(const WeightsView &w, const __nv_bfloat16 *x, int64_t batch,
                   int64_t ldx, float *y, int64_t ldy, cudaStream_t stream) {
  const int sms = device_sms();
  switch (batch) {
    case 1:
      if (pick_rows(w.n, w.k, 16, 16, sms) == 4)
        return launch_cfg<1, 16, 4, 2, 512>(w, x, ldx, y, ldy, sms, stream);
      return launch_cfg<1, 16, 2, 3, 512>(w, x, ldx, y, ldy, sms, stream);
    case 2:
      return launch_cfg<2, 16, 2, 2, 512>(w, x, ldx, y, ldy, sms, stream);
    case 3:
      return launch_cfg<3, 8, 2, 3, 512>(w, x, ldx, y, ldy, sms, stream);
    default:
      return launch_cfg<4, 8, 2, 3, 512>(w, x, ldx, y, ldy, sms, stream);
  }
}

}  // namespace tq
