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
//   - Codes stream through a per-warp ring of shared-memory stages filled by
//     cp.async (16 B per lane and row, L2 only), several row groups ahead of
//     the math and continuously across chunks. Each lane reads back exactly
//     the bytes its own copies wrote.
//   - x for the warp's chunk is converted once to fp32 and kept in registers
//     while the warp walks the CTA's rows, R rows at a time; the next chunk's
//     x is fetched one row group early.
//   - The code book is replicated once per lane in shared memory: entry e of
//     lane l's copy sits at byte e*128 + 4*l (all 256 byte values, so an
//     invalid code reads its NaN entry): a warp's 32 random lookups hit 32
//     distinct banks.
//   - Products accumulate in fp32 with packed FFMA2 over k pairs; per row
//     group the R*B partial sums are reduced across lanes with a transposing
//     butterfly (about 2 shuffles per value instead of 5), summed over the
//     warp's chunks in shared memory, then over warps in a fixed order:
//     deterministic.
#include "tq_common.cuh"
#include "tq_linear.cuh"

namespace tq {
namespace {

constexpr int kLutStride = 128;              // bytes per code-book entry
constexpr int kLutBytes = 256 * kLutStride;  // all byte values: 32 KB
constexpr int kMaxWarps = 8;
constexpr int kCtasPerSm = 2;
constexpr int kStages = 4;                   // row groups in flight per warp

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// Asynchronous global -> shared copy of BYTES (16 or 8) bytes; src_size 0
// writes zeros and reads nothing.
template <int BYTES>
__device__ __forceinline__ void cp_async(uint32_t dst, const void *src,
                                         bool valid) {
  const int n = valid ? BYTES : 0;
  if constexpr (BYTES == 16) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst),
                 "l"(src), "r"(n)
                 : "memory");
  } else {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(dst),
                 "l"(src), "r"(n)
                 : "memory");
  }
}

__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// bf16 pair (low half = lower k) -> float2.
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

// Code-book value of byte q of word w for this lane (lane8 = 8 * lane): the
// byte permute yields code*256 + 8*lane, halved to code*128 + 4*lane.
__device__ __forceinline__ float lut_at(const uint8_t *lut_smem, uint32_t w,
                                        int q, uint32_t lane8) {
  const uint32_t a2 = __byte_perm(w, lane8, 0x5504u | ((uint32_t)q << 4));
  return *reinterpret_cast<const float *>(lut_smem + (a2 >> 1));
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
struct Rows {  // rows per group
  static constexpr int value = (B <= 2) ? 4 : 2;
};

template <int B, int KPL>
struct GemvBShape {
  static constexpr int R = Rows<B>::value;
  static constexpr int M = pow2_ceil(R * B);  // values reduced per group
  static constexpr int KC = 32 * KPL;         // k per warp chunk
  static constexpr int NW = KPL / 4;          // code words per lane per row
  static constexpr int SLOT = R * 32 * KPL;   // ring-slot bytes per warp
  static constexpr int RING = kStages * SLOT; // ring bytes per warp
};

template <int B, int KPL>
__global__ void __launch_bounds__(kMaxWarps * 32, kCtasPerSm)
    gemv_b_kernel(const uint8_t *__restrict__ codes, int64_t n, int64_t k,
                  const float *__restrict__ lut,
                  const uint16_t *__restrict__ rho, int rps,
                  const __nv_bfloat16 *__restrict__ x, int64_t ldx,
                  float *__restrict__ y, int64_t ldy, int rows_max) {
  using S = GemvBShape<B, KPL>;
  constexpr int R = S::R, M = S::M, KC = S::KC, NW = S::NW;
  extern __shared__ __align__(16) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  uint8_t *ring = smem + kLutBytes + warp * S::RING;
  float *red = reinterpret_cast<float *>(smem + kLutBytes + nwarps * S::RING);

  const int64_t row_lo = (int64_t)blockIdx.x * n / gridDim.x;
  const int rows = (int)((int64_t)(blockIdx.x + 1) * n / gridDim.x - row_lo);
  const uint8_t *crow = codes + row_lo * k;
  const int64_t nchunks = (k + KC - 1) / KC;
  const int nc_w = (int)((nchunks - warp + nwarps - 1) / nwarps);  // my chunks
  const int ng = (rows + R - 1) / R;                               // row groups
  const int total = nc_w * ng;

  // Issue the copies of item i (chunk i / ng, row group i % ng) into its slot.
  auto issue = [&](int i) {
    const int ci = i / ng, g = i % ng;
    const int64_t kb = (warp + (int64_t)ci * nwarps) * KC + (int64_t)lane * KPL;
    const bool lane_ok = kb < k;
    const uint32_t dst = smem_addr(ring + (i % kStages) * S::SLOT) + lane * KPL;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int row = g * R + r;
      const bool ok = lane_ok && row < rows;
      cp_async<KPL>(dst + r * 32 * KPL, ok ? crow + (int64_t)row * k + kb : codes,
                    ok);
    }
  };
  // Raw bf16 words of x for chunk ci (this lane's KPL columns).
  uint32_t xr[B][KPL / 2];
  auto load_x = [&](int ci) {
    const int64_t kb = (warp + (int64_t)ci * nwarps) * KC + (int64_t)lane * KPL;
#pragma unroll
    for (int b = 0; b < B; ++b) {
#pragma unroll
      for (int i = 0; i < KPL / 2; i += 4) {
        uint4 v = make_uint4(0, 0, 0, 0);
        if (ci < nc_w && kb < k)
          v = *reinterpret_cast<const uint4 *>(x + b * ldx + kb + 2 * i);
        xr[b][i] = v.x;
        xr[b][i + 1] = v.y;
        xr[b][i + 2] = v.z;
        xr[b][i + 3] = v.w;
      }
    }
  };

  // Start the code stream and the first x before building the code book.
#pragma unroll
  for (int p = 0; p < kStages - 1; ++p) {
    if (p < total) issue(p);
    cp_async_commit();
  }
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
  for (int i = threadIdx.x; i < nwarps * rows_max * B; i += blockDim.x)
    red[i] = 0.0f;
  __syncthreads();

  const uint32_t lane8 = (uint32_t)lane * 8u;
  float2 xv[B][KPL / 2];
  bool lane_ok = false;
  for (int i = 0; i < total; ++i) {
    if (i + kStages - 1 < total) issue(i + kStages - 1);
    cp_async_commit();
    cp_async_wait<kStages - 1>();  // item i's copies have landed
    const int ci = i / ng, g = i % ng;
    if (g == 0) {
      const int64_t kb =
          (warp + (int64_t)ci * nwarps) * KC + (int64_t)lane * KPL;
      lane_ok = kb < k;
#pragma unroll
      for (int b = 0; b < B; ++b)
#pragma unroll
        for (int q = 0; q < KPL / 2; ++q) xv[b][q] = bf16x2_to_float2(xr[b][q]);
      load_x(ci + 1);  // next chunk's x, consumed ng groups later
    }
    float2 acc[R][B];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int b = 0; b < B; ++b) acc[r][b] = make_float2(0.f, 0.f);
    if (lane_ok) {
      const uint8_t *slot = ring + (i % kStages) * S::SLOT + lane * KPL;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        uint32_t cw[NW];
        if constexpr (KPL == 16) {
          const uint4 v = *reinterpret_cast<const uint4 *>(slot + r * 32 * KPL);
          cw[0] = v.x; cw[1] = v.y; cw[2] = v.z; cw[3] = v.w;
        } else {
          const uint2 v = *reinterpret_cast<const uint2 *>(slot + r * 32 * KPL);
          cw[0] = v.x; cw[1] = v.y;
        }
#pragma unroll
        for (int wi = 0; wi < NW; ++wi) {
#pragma unroll
          for (int q = 0; q < 4; q += 2) {
            const float2 wv = make_float2(lut_at(smem, cw[wi], q, lane8),
                                          lut_at(smem, cw[wi], q + 1, lane8));
#pragma unroll
            for (int b = 0; b < B; ++b)
              acc[r][b] = __ffma2_rn(wv, xv[b][wi * 2 + q / 2], acc[r][b]);
          }
        }
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
      const int r = idx / B, b = idx % B;
      const int row = g * R + r;
      if (row < rows) red[(warp * rows_max + row) * B + b] += s;
    }
  }
  cp_async_wait<0>();
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

ChunkPlan plan_chunks(int64_t k) {
  ChunkPlan best{8, 1};
  double best_eff = -1.0;
  for (int kpl = 16; kpl >= 8; kpl /= 2) {
    const int64_t nchunks = (k + 32 * kpl - 1) / (32 * kpl);
    const int wmax = (int)(nchunks < kMaxWarps ? nchunks : kMaxWarps);
    for (int w = wmax; w >= 1 && w >= wmax - 4; --w) {
      const int64_t rounds = (nchunks + w - 1) / w;
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
  using S = GemvBShape<B, KPL>;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  constexpr int kMaxRedBytes = 16 * 1024;
  const int64_t rows_cap = kMaxRedBytes / (warps * B * 4);
  int64_t ctas = (int64_t)sms * kCtasPerSm;
  if ((w.n + ctas - 1) / ctas > rows_cap) ctas = (w.n + rows_cap - 1) / rows_cap;
  if (ctas > w.n) ctas = w.n;
  const int rows_max = (int)((w.n + ctas - 1) / ctas);
  const size_t smem = kLutBytes + (size_t)warps * S::RING +
                      (size_t)warps * rows_max * B * sizeof(float);
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
  const ChunkPlan p = plan_chunks(w.k);
  if (p.kpl == 16) return launch_kpl<B, 16>(w, x, ldx, y, ldy, p.warps, stream);
  return launch_kpl<B, 8>(w, x, ldx, y, ldy, p.warps, stream);
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
