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
//     packed fp32x2 FMA (even and odd k accumulate separately).
//   - Work unit: R rows x one k-chunk of 512 codes (16 per lane, a fully
//     coalesced 512-byte run per row). A CTA (one per SM) owns an even share
//     of the rows; its units are ordered row-group major and cut into equal
//     contiguous ranges, one per warp, so every warp does the same amount of
//     work (+-1 unit) and streams along its rows.
//   - HBM needs tens of KB in flight per SM. The codes therefore stream
//     through a per-warp ring of D unit slots in shared memory, filled by
//     asynchronous 16-byte copies (each lane copies, and later reads back,
//     only its own bytes, so no barrier is involved); D-1 units are in
//     flight while one is computed, without holding registers. The rings
//     live in the shared memory around the code book. x is read through
//     the caches (L2, and L1 where it fits), one unit ahead.
//   - Sums stay in registers along a row segment; at its end the R*B values
//     are reduced across lanes by a transposing butterfly and stored in the
//     slot of the segment's first chunk. The slots of a row are added in a
//     fixed order at the end, so the result does not depend on timing.
#include "tq_common.cuh"
#include "tq_linear.cuh"

namespace tq {
namespace {

constexpr uint32_t kLutAddr = 0x10000u;  // shared-window address of the book
constexpr uint32_t kLutStride = 256;     // bytes per entry (32 lane copies)
constexpr uint32_t kRedAddr = 0x20000u;  // partial sums follow the book
constexpr int kSmemMax = 227 * 1024;     // dynamic shared memory per CTA
// Rings below the code book start at or below this shared-window address
// (the dynamic window starts right after the 1 KB reserved per CTA).
constexpr uint32_t kRingLoAddr = 0x1000u;
constexpr int KPL = 16;             // codes per lane and row
constexpr int KC = 32 * KPL;        // codes per chunk
constexpr uint32_t kRowBytes = KC;  // one row of a unit slot

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src,
                                           uint32_t n) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst),
               "l"(src), "r"(n)
               : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// x: read-only and shared by every row (cached loads). Volatile so that it
// stays where it is issued, a unit ahead of its use.
__device__ __forceinline__ uint4 ld_x16(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 lds_v4(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a)
               : "memory");
  return v;
}

// Code-book lookup. Not volatile, so the compiler may schedule it freely; it
// is ordered after the code book is built through its address operand.
__device__ __forceinline__ float lds_f32(uint32_t a) {
  float v;
  asm("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}

__device__ __forceinline__ float lds_f32_volatile(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
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

// Position of a work unit: row group g and chunk c.
struct UnitPos {
  int g, c;
};

__device__ __forceinline__ void advance(UnitPos &q, int nchunks) {
  if (++q.c == nchunks) {
    q.c = 0;
    ++q.g;
  }
}

__device__ __forceinline__ void advance_cm(UnitPos &q, int ng) {
  if (++q.g == ng) {
    q.g = 0;
    ++q.c;
  }
}

// hi_ring: shared-window address of the rings placed above the partial sums.
// CM (chunk-major): units ordered chunk first, so a warp keeps one chunk's x
// (converted once) in registers across the row groups it walks and reduces
// every unit (the dispatched order: converting x per unit costs more than the
// reductions). Otherwise row-group major: sums stay in registers along a row
// segment and are reduced once per segment.
template <int B, int R, int D, int NT, bool CM>
__global__ void __launch_bounds__(NT, 1)
    gemv_b_kernel(const uint8_t *__restrict__ codes, int64_t n, int64_t k,
                  const float *__restrict__ lut,
                  const uint16_t *__restrict__ rho, int rps,
                  const __nv_bfloat16 *__restrict__ x, int64_t ldx,
                  float *__restrict__ y, int64_t ldy, int rows_max,
                  uint32_t hi_ring) {
  constexpr int NW = KPL / 4;          // code words per lane and row
  constexpr int NX = KPL / 2;          // x words (bf16 pairs) per lane and row
  constexpr int M = pow2_ceil(R * B);  // values reduced per row segment
  constexpr int kWarps = NT / 32;
  constexpr uint32_t kSlot = R * kRowBytes;  // one unit's codes
  constexpr uint32_t kRing = D * kSlot;      // one warp's ring
  extern __shared__ __align__(16) uint8_t smem[];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row_lo = (int64_t)blockIdx.x * n / gridDim.x;
  const int rows = (int)((int64_t)(blockIdx.x + 1) * n / gridDim.x - row_lo);
  // the next kernel on the stream may be scheduled onto SMs this grid frees
  pdl_launch_dependents();

  // The layout assumes the dynamic window starts at or below kRingLoAddr
  // (then the request covers the code book, the partial sums and the rings).
  const uint32_t base = (uint32_t)__cvta_generic_to_shared(smem);
  if (base > kRingLoAddr) {
    pdl_wait();
    for (int i = threadIdx.x; i < rows * B; i += NT) {
      const int r = i / B, b = i - r * B;
      y[(int64_t)b * ldy + row_lo + r] = __int_as_float(0x7FC00000);
    }
    return;
  }
  const uint32_t lo_ring = (base + 127u) & ~127u;
  const int lo_warps = (int)((kLutAddr - lo_ring) / kRing);
  const uint32_t ring = warp < lo_warps
                            ? lo_ring + (uint32_t)warp * kRing
                            : hi_ring + (uint32_t)(warp - lo_warps) * kRing;
  const uint32_t ring_end = ring + kRing;
  const uint32_t lane16 = (uint32_t)lane * 16u;

  const int ng = (rows + R - 1) / R;
  const int nchunks = (int)((k + KC - 1) / KC);
  const int units = ng * nchunks;  // u = g * nchunks + c (CM: c * ng + g)
  const int u_begin = (int)((int64_t)units * warp / kWarps);
  const int u_end = (int)((int64_t)units * (warp + 1) / kWarps);
  const int64_t kstride = k;
  const int64_t group_step = (int64_t)R * kstride;
  const uint8_t *crow = codes + row_lo * kstride + lane * KPL;
  const __nv_bfloat16 *xl = x + lane * KPL;
  // lanes past k in the last chunk hold nothing
  const bool last_ok = (int64_t)(nchunks - 1) * KC + lane * KPL < k;

  UnitPos ld;  // next unit whose codes are copied
  if constexpr (CM) {
    ld.c = u_begin / ng;
    ld.g = u_begin - ld.c * ng;
  } else {
    ld.g = u_begin / nchunks;
    ld.c = u_begin - ld.g * nchunks;
  }
  const uint8_t *ld_p = crow + (int64_t)ld.g * group_step + (int64_t)ld.c * KC;
  int u_ld = u_begin;
  uint32_t ld_slot = ring;
  UnitPos cur = ld;

  // Copy unit u_ld's codes into the next ring slot (one commit group per
  // unit, empty past the range). Rows past the CTA's rows and lanes past k
  // are zero-filled; their products are never used.
  auto issue = [&]() {
    if (u_ld < u_end) {
      const uint32_t dst = ld_slot + lane16;
      const bool full =
          (ld.g + 1) * R <= rows && (int64_t)(ld.c + 1) * KC <= k;  // uniform
      if (full) {
#pragma unroll
        for (int r = 0; r < R; ++r)
          cp_async16(dst + r * kRowBytes, ld_p + r * kstride, 16u);
      } else {
        const bool ok = ld.c + 1 < nchunks || last_ok;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const bool okr = ok && ld.g * R + r < rows;
          cp_async16(dst + r * kRowBytes, okr ? ld_p + r * kstride : codes,
                     okr ? 16u : 0u);
        }
      }
      if constexpr (CM) {
        advance_cm(ld, ng);
        ld_p = ld.g == 0 ? crow + (int64_t)ld.c * KC : ld_p + group_step;
      } else {
        advance(ld, nchunks);
        ld_p = ld.c == 0 ? crow + (int64_t)ld.g * group_step : ld_p + KC;
      }
    }
    cp_async_commit();
    ld_slot = ld_slot + kSlot == ring_end ? ring : ld_slot + kSlot;
    ++u_ld;
  };

  // Raw bf16 x of chunk c for this lane (zero past k).
  uint32_t xw[B][NX];
  auto load_x = [&](int c) {
    const bool ok = c + 1 < nchunks || last_ok;
    const __nv_bfloat16 *xp = xl + (int64_t)c * KC;
#pragma unroll
    for (int b = 0; b < B; ++b)
#pragma unroll
      for (int q = 0; q < NX; q += 4) {
        uint4 v = make_uint4(0, 0, 0, 0);
        if (ok) v = ld_x16(xp + b * ldx + 2 * q);
        xw[b][q] = v.x;
        xw[b][q + 1] = v.y;
        xw[b][q + 2] = v.z;
        xw[b][q + 3] = v.w;
      }
  };

  // While the kernel before this one on the stream finishes: warm L2 with
  // this warp's first units (about 8 KB; lane r < R takes row r of each),
  // then wait for that kernel's completion before reading user memory.
  {
    constexpr int kPre = (8192 / (int)kSlot) > 1 ? 8192 / (int)kSlot : 1;
    UnitPos pq = ld;
    const uint8_t *pp = ld_p;
    for (int i = 0; i < kPre && u_begin + i < u_end; ++i) {
      const int64_t k0 = (int64_t)pq.c * KC;
      const uint32_t run = (uint32_t)(k - k0 < KC ? k - k0 : KC);
      if (lane < R && pq.g * R + lane < rows)
        prefetch_l2_bulk(pp - lane * KPL + (int64_t)lane * kstride, run);
      if constexpr (CM) {
        advance_cm(pq, ng);
        pp = pq.g == 0 ? crow + (int64_t)pq.c * KC : pp + group_step;
      } else {
        advance(pq, nchunks);
        pp = pq.c == 0 ? crow + (int64_t)pq.g * group_step : pp + KC;
      }
    }
  }
  pdl_wait();

  // Start the first copies, then clear the partial sums and build the code
  // book while they fly.
#pragma unroll
  for (int d = 0; d < D - 1; ++d) issue();
  if constexpr (!CM) load_x(cur.c);
  const int red_words = nchunks * rows_max * B;
  for (int i = threadIdx.x; i < red_words; i += NT)
    sts_f32(kRedAddr + 4u * (uint32_t)i, 0.0f);
  for (int i = threadIdx.x; i < 256 * 8; i += NT) {
    const int e = i >> 3, j = i & 7;
    sts_v4(kLutAddr + e * kLutStride + j * 16, __ldg(lut + e));
  }
  __syncthreads();
  // Defined after the barrier (volatile), so no table lookup can be hoisted
  // above it.
  uint32_t lane_lut;
  asm volatile("mov.b32 %0, %1;" : "=r"(lane_lut) : "r"(kLutAddr | (lane << 2)));

  float2 acc[R][B];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int b = 0; b < B; ++b) acc[r][b] = make_float2(0.0f, 0.0f);
  int c_seg = cur.c;  // first chunk of the current row segment
  uint32_t cur_slot = ring;
  float2 xv[B][NX];  // x of the current chunk (CM: kept across units)
  int xc = -1;       // chunk whose x is in xv (CM)

  for (int u = u_begin; u < u_end; ++u) {
    issue();                 // unit u + D - 1
    cp_async_wait<D - 1>();  // unit u has landed
    uint32_t cw[R][NW];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const uint4 v = lds_v4(cur_slot + r * kRowBytes + lane16);
      cw[r][0] = v.x; cw[r][1] = v.y; cw[r][2] = v.z; cw[r][3] = v.w;
    }
    cur_slot = cur_slot + kSlot == ring_end ? ring : cur_slot + kSlot;

    auto convert_x = [&]() {
#pragma unroll
      for (int b = 0; b < B; ++b)
#pragma unroll
        for (int q = 0; q < NX; ++q)
          xv[b][q] = make_float2(__uint_as_float(xw[b][q] << 16),
                                 __uint_as_float(xw[b][q] & 0xFFFF0000u));
    };
    if constexpr (CM) {
      if (cur.c != xc) {  // entering a chunk: fetch and convert its x once
        xc = cur.c;
        load_x(xc);
        convert_x();
      }
    } else {
      convert_x();
      if (u + 1 < u_end) load_x(cur.c + 1 == nchunks ? 0 : cur.c + 1);
    }

    if (cur.c + 1 < nchunks || last_ok) {
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

    if (CM || u + 1 == u_end || cur.c + 1 == nchunks) {
      if constexpr (CM) c_seg = cur.c;  // every unit is its own segment
      // End of a row segment: reduce across lanes and store the sums in the
      // slot of the segment's first chunk (distinct for every warp touching
      // the rows).
      float v[M];
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int b = 0; b < B; ++b) {
          v[r * B + b] = acc[r][b].x + acc[r][b].y;
          acc[r][b] = make_float2(0.0f, 0.0f);
        }
#pragma unroll
      for (int q = R * B; q < M; ++q) v[q] = 0.0f;
      const float s = butterfly_reduce<M>(v, lane);
      constexpr int kLow = 32 / M;  // lanes holding the same reduced value
      const int idx = lane / kLow;
      if ((lane % kLow) == 0 && idx < R * B) {
        const int r = idx / B, b = idx - (idx / B) * B;
        const int row = cur.g * R + r;
        if (row < rows)
          sts_f32(
              kRedAddr + (uint32_t)(((c_seg * rows_max + row) * B + b) * 4),
              s);
      }
      c_seg = 0;  // the next unit starts a row group at chunk 0
    }
    if constexpr (CM) {
      advance_cm(cur, ng);
    } else {
      advance(cur, nchunks);
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // Sum each row's chunk slots in a fixed order: lane-strided, then across
  // the warp.
  for (int o = warp; o < rows * B; o += kWarps) {
    const int r = o / B, b = o - r * B;
    float s = 0.0f;
    for (int c = lane; c < nchunks; c += 32)
      s += lds_f32_volatile(
          kRedAddr + (uint32_t)(((c * rows_max + r) * B + b) * 4));
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, m);
    if (lane == 0) {
      const int64_t row = row_lo + r;
      const float scale =
          rho ? __half2float(__ushort_as_half(rho[row / rps])) : 1.0f;
      y[(int64_t)b * ldy + row] = scale * s;
    }
  }
}

template <int B, int R, int D, int NT, bool CM = false>
cudaError_t launch_cfg(const WeightsView &w, const __nv_bfloat16 *x,
                       int64_t ldx, float *y, int64_t ldy, int sms,
                       cudaStream_t stream) {
  constexpr int kWarps = NT / 32;
  constexpr uint32_t kRing = D * R * kRowBytes;
  // Rings that fit below the code book even with the window at kRingLoAddr;
  // the others go above the partial sums.
  constexpr int lo_min = (int)((kLutAddr - kRingLoAddr) / kRing);
  constexpr int hi_warps = kWarps > lo_min ? kWarps - lo_min : 0;
  const int64_t nchunks = (w.k + KC - 1) / KC;
  int64_t ctas = sms < w.n ? sms : w.n;
  // the partial sums (one slot per chunk, row and batch row) must fit
  // between the code book and the upper rings
  const int64_t red_max =
      (int64_t)kSmemMax - kRedAddr - (int64_t)hi_warps * kRing - 128;
  const int64_t rows_cap = red_max / (nchunks * B * 4);
  if (rows_cap < 1) return cudaErrorInvalidValue;
  if ((w.n + ctas - 1) / ctas > rows_cap) ctas = (w.n + rows_cap - 1) / rows_cap;
  const int rows_max = (int)((w.n + ctas - 1) / ctas);
  const uint32_t red_bytes = (uint32_t)(nchunks * rows_max * B * 4);
  const uint32_t hi_ring = (kRedAddr + red_bytes + 127u) & ~127u;
  const size_t smem = hi_ring + (size_t)hi_warps * kRing;
  if (smem > (size_t)kSmemMax) return cudaErrorInvalidValue;
  auto kern = gemv_b_kernel<B, R, D, NT, CM>;
  cudaError_t e = ensure_smem_limit<gemv_b_kernel<B, R, D, NT, CM>>(kSmemMax);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3((unsigned)ctas), dim3(NT), smem, stream,
                    w.codes, w.n, w.k, w.lut, w.scales, w.rps, x, ldx, y, ldy,
                    rows_max, hi_ring);
}

int device_sms() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

}  // namespace

bool gemv_b_supported(const WeightsView &w, int64_t batch) {
  // one code book per layer: the kernel keeps it lane-replicated on chip
  return w.format == TQ_FMT_B && w.lut_rows == 0 && batch >= 1 && batch <= 4;
}

cudaError_t gemv_b(const WeightsView &w, const __nv_bfloat16 *x, int64_t batch,
                   int64_t ldx, float *y, int64_t ldy, cudaStream_t stream) {
  // The kernel places its code book and rings at fixed shared-window
  // addresses, which assumes the dynamic window starts at or below
  // kRingLoAddr (the per-CTA reserved shared memory comes first). Refuse a
  // device where it would not, instead of launching a kernel that could only
  // write NaN.
  int dev = 0, reserved = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock,
                             dev);
  if (e != cudaSuccess) return e;
  if ((uint32_t)reserved > kRingLoAddr) return cudaErrorNotSupported;
  const int sms = device_sms();
  switch (batch) {
    case 1: return launch_cfg<1, 8, 2, 512, true>(w, x, ldx, y, ldy, sms, stream);
    case 2: return launch_cfg<2, 4, 4, 512, true>(w, x, ldx, y, ldy, sms, stream);
    case 3: return launch_cfg<3, 2, 4, 512, true>(w, x, ldx, y, ldy, sms, stream);
    default: return launch_cfg<4, 2, 4, 512, true>(w, x, ldx, y, ldy, sms, stream);
  }
}

}  // namespace tq
