// Format B fused GEMV, batch 1 and 2, row-parallel lanes (alphaneural.io
// page, sections 3.2, 3.3 and 4.2):
//   y[b][n] = rho[n / rps] * sum_k LUT[code[n][k]] * x[b][k].
//
// Memory-bound at one code byte per weight; the design keeps the issued
// instructions per weight near three (a byte permute that is the whole
// shared address, one shared load, one FFMA) so that issue never binds:
//   - One CTA per SM owns rows [i*n/P, (i+1)*n/P). A warp owns RPW rows: its
//     lanes are RPW rows x KP k-parts, each lane reading 16 consecutive codes,
//     so every row gets a contiguous 16*KP bytes per step (coalesced) and the
//     warp walks the whole of K with U steps of code loads in flight. The
//     only cross-lane work is log2(KP) shuffles per row at the very end.
//   - x is staged once per CTA in shared memory as fp32, permuted so the KP
//     k-parts of a step read consecutive 16-byte chunks (conflict-free, rows
//     of the same part broadcast).
//   - The code book is replicated once per lane (entry e of lane l's copy at
//     byte e*256 + 4*l; all 256 byte values, so invalid codes read NaN) and
//     placed at a 64 KB-aligned shared address: then the byte permute of the
//     code word with (page << 16 | 4*l) is the complete address. If the
//     alignment cannot be had, one add restores the base.
#include "tq_common.cuh"
#include "tq_linear.cuh"

namespace tq {
namespace {

constexpr int kLutBytes = 256 * 256;  // 256 entries x 32 lane copies x 4 B
constexpr int kReservedSmem = 1024;   // per-CTA system shared memory (sm_100)
constexpr int kThreads = 1024;

__device__ __forceinline__ uint4 ld_stream16(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ float4 lds_f32x4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
  return v;
}

// Shared-memory layout: x (fp32, permuted, padded to whole steps) first, then
// the code book at the first offset whose shared address is 64 KB aligned
// (computed for the usual base; the kernel checks it).
struct RowsLayout {
  int64_t x_bytes;
  int64_t red_off;
  int64_t lut_off;
  int64_t total;
};

template <int B, int KP>
RowsLayout rows_layout(int64_t k, int64_t red_bytes) {
  const int64_t step = 16 * KP;
  const int64_t kpad = (k + step - 1) / step * step;
  RowsLayout L;
  L.x_bytes = kpad * B * 4;
  L.red_off = L.x_bytes;
  const int64_t used = L.x_bytes + red_bytes;
  const int64_t base = kReservedSmem;
  L.lut_off = ((base + used + 65535) / 65536) * 65536 - base;
  L.total = L.lut_off + kLutBytes;
  return L;
}

template <int B, int RPW, int U, bool PAGED>
__device__ __forceinline__ void walk_rows(
    const uint8_t *__restrict__ cp, bool row_ok, int k32, int s_begin,
    int s_end, int p, uint32_t xs, uint32_t perm_op, uint32_t fix,
    uint32_t (&c)[U][4], float (&acc)[B]) {
  constexpr int KP = 32 / RPW;
  constexpr int STEP = 16 * KP;
  auto load = [&](int s, uint32_t(&cc)[4]) {
    cc[0] = cc[1] = cc[2] = cc[3] = 0x79797979u;  // code 121: weight 0
    if (row_ok && s < s_end && s * STEP + p * 16 < k32) {
      const uint4 v = ld_stream16(cp + s * STEP);
      cc[0] = v.x; cc[1] = v.y; cc[2] = v.z; cc[3] = v.w;
    }
  };
  for (int s0 = s_begin; s0 < s_end; s0 += U) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int s = s0 + u;
      if (s < s_end) {
        const uint32_t cur[4] = {c[u][0], c[u][1], c[u][2], c[u][3]};
        load(s + U, c[u]);
        const uint32_t xa = xs + (uint32_t)((s * 4 * KP + p) * B * 16);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float xv[B][4];
#pragma unroll
          for (int b = 0; b < B; ++b) {
            const float4 t = lds_f32x4(xa + (q * KP * B + b) * 16);
            xv[b][0] = t.x; xv[b][1] = t.y; xv[b][2] = t.z; xv[b][3] = t.w;
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t a =
                __byte_perm(cur[q], perm_op, 0x7604u | ((uint32_t)e << 4));
            const float wv = lds_f32(PAGED ? a : a + fix);
#pragma unroll
            for (int b = 0; b < B; ++b) acc[b] = fmaf(wv, xv[b][e], acc[b]);
          }
        }
      }
    }
  }
}

// Warps are WK k-slices x WR row blocks of RPW rows; red holds the partial
// sums [WK][rows][B].
template <int B, int RPW, int U>
__global__ void __launch_bounds__(kThreads, 1)
    gemv_b_rows_kernel(const uint8_t *__restrict__ codes, int64_t n,
                       int64_t k, const float *__restrict__ lut,
                       const uint16_t *__restrict__ rho, int rps,
                       const __nv_bfloat16 *__restrict__ x, int64_t ldx,
                       float *__restrict__ y, int64_t ldy, int lut_off,
                       int red_off, int wk_count, int rows_max) {
  constexpr int KP = 32 / RPW;    // k-parts (lanes) per row
  constexpr int STEP = 16 * KP;   // k per warp step
  extern __shared__ __align__(16) uint8_t smem[];
  const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(smem);
  const uint32_t xs = sbase;                          // permuted fp32 x
  const uint32_t lut_addr = sbase + (uint32_t)lut_off;
  float *red = reinterpret_cast<float *>(smem + red_off);
  const int k32 = (int)k;
  const int nsteps = (k32 + STEP - 1) / STEP;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int wr_count = nwarps / wk_count;
  const int wk = warp / wr_count, wr = warp % wr_count;
  const int r = lane / KP, p = lane % KP;
  const int64_t row_lo = (int64_t)blockIdx.x * n / gridDim.x;
  const int rows = (int)((int64_t)(blockIdx.x + 1) * n / gridDim.x - row_lo);
  const int nblk = (rows + RPW - 1) / RPW;
  const int s_begin = nsteps * wk / wk_count;
  const int s_end = nsteps * (wk + 1) / wk_count;

  // First code loads of this warp's first row block, before any staging.
  uint32_t c[U][4];
  auto first_loads = [&](int blk) {
    const int row = blk * RPW + r;
    const bool ok = row < rows;
    const uint8_t *cp = codes + (row_lo + (ok ? row : 0)) * k + p * 16;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int s = s_begin + u;
      c[u][0] = c[u][1] = c[u][2] = c[u][3] = 0x79797979u;
      if (ok && s < s_end && s * STEP + p * 16 < k32) {
        const uint4 v = ld_stream16(cp + s * STEP);
        c[u][0] = v.x; c[u][1] = v.y; c[u][2] = v.z; c[u][3] = v.w;
      }
    }
  };
  if (wr < nblk) first_loads(wr);

  // Stage x, 8 elements (16 bytes) per load: element k of batch b goes to
  // float index ((s*4 + q)*KP + p)*4*B + b*4 + i, k = s*STEP + p*16 + q*4 + i,
  // so a lane's four chunks of a step are 16-byte loads at stride KP*16*B.
  float *xsp = reinterpret_cast<float *>(smem);
  const int nvec = nsteps * STEP / 8;
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    const int kk = v * 8;
    const int s = kk / STEP, rem = kk % STEP;
    const int pp = rem >> 4, q0 = (rem >> 2) & 3;  // q0 even: two chunks
#pragma unroll
    for (int b = 0; b < B; ++b) {
      uint4 raw = make_uint4(0, 0, 0, 0);
      if (kk < k32) raw = *reinterpret_cast<const uint4 *>(x + b * ldx + kk);
      const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float4 f;
        f.x = __uint_as_float(wd[2 * h] << 16);
        f.y = __uint_as_float(wd[2 * h] & 0xFFFF0000u);
        f.z = __uint_as_float(wd[2 * h + 1] << 16);
        f.w = __uint_as_float(wd[2 * h + 1] & 0xFFFF0000u);
        const int idx = (((s * 4 + q0 + h) * KP + pp) * B + b) * 4;
        *reinterpret_cast<float4 *>(xsp + idx) = f;
      }
    }
  }
  // Replicate the code book with conflict-free rotated 16-byte stores.
  for (int e = threadIdx.x; e < 256; e += blockDim.x) {
    const float v = __ldg(lut + e);
    const float4 v4 = make_float4(v, v, v, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int jj = (j + e) & 7;
      *reinterpret_cast<float4 *>(smem + lut_off + e * 256 + jj * 16) = v4;
    }
  }
  __syncthreads();

  // Byte-permute operand: lane copy offset in byte 0, the 64 KB page of the
  // table in bytes 2-3; without the page trick one add restores the base.
  const bool paged = (lut_addr & 0xFFFFu) == 0;
  const uint32_t perm_op =
      (paged ? (lut_addr & 0xFFFF0000u) : 0u) | ((uint32_t)lane * 4u);
  for (int blk = wr; blk < nblk; blk += wr_count) {
    if (blk != wr) first_loads(blk);
    const int row = blk * RPW + r;
    const bool row_ok = row < rows;
    const uint8_t *cp = codes + (row_lo + (row_ok ? row : 0)) * k + p * 16;
    float acc[B];
#pragma unroll
    for (int b = 0; b < B; ++b) acc[b] = 0.0f;
    if (paged)
      walk_rows<B, RPW, U, true>(cp, row_ok, k32, s_begin, s_end, p, xs,
                                 perm_op, 0u, c, acc);
    else
      walk_rows<B, RPW, U, false>(cp, row_ok, k32, s_begin, s_end, p, xs,
                                  perm_op, lut_addr, c, acc);
#pragma unroll
    for (int b = 0; b < B; ++b) {
#pragma unroll
      for (int o = KP / 2; o >= 1; o >>= 1)
        acc[b] += __shfl_xor_sync(0xFFFFFFFFu, acc[b], o);
    }
    if (p == 0 && row_ok) {
#pragma unroll
      for (int b = 0; b < B; ++b) red[(wk * rows_max + row) * B + b] = acc[b];
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < rows * B; i += blockDim.x) {
    const int rr = i / B, b = i % B;
    float sum = 0.0f;
    for (int w = 0; w < wk_count; ++w) sum += red[(w * rows_max + rr) * B + b];
    const int64_t grow = row_lo + rr;
    const float scale =
        rho ? __half2float(__ushort_as_half(rho[grow / rps])) : 1.0f;
    y[(int64_t)b * ldy + grow] = scale * sum;
  }
}

struct RowsPlan {
  int64_t ctas;
  int rows_max;
  int wk;
  int wr;
};

template <int RPW>
RowsPlan plan_rows(int64_t n, int64_t k, int sms) {
  constexpr int KP = 32 / RPW;
  RowsPlan P;
  P.ctas = sms < n ? sms : n;
  P.rows_max = (int)((n + P.ctas - 1) / P.ctas);
  const int nblk = (P.rows_max + RPW - 1) / RPW;
  const int nsteps = (int)((k + 16 * KP - 1) / (16 * KP));
  const int max_warps = kThreads / 32;
  const int rounds = (nblk + max_warps - 1) / max_warps;  // blocks per warp
  P.wr = (nblk + rounds - 1) / rounds;
  P.wk = max_warps / P.wr;
  if (P.wk > nsteps) P.wk = nsteps;
  if (P.wk < 1) P.wk = 1;
  return P;
}

template <int B, int RPW>
cudaError_t launch_rows(const WeightsView &w, const __nv_bfloat16 *x,
                        int64_t ldx, float *y, int64_t ldy, int sms,
                        cudaStream_t stream) {
  constexpr int KP = 32 / RPW;
  constexpr int U = 8;
  const RowsPlan P = plan_rows<RPW>(w.n, w.k, sms);
  const RowsLayout L =
      rows_layout<B, KP>(w.k, (int64_t)P.wk * P.rows_max * B * 4);
  auto kern = gemv_b_rows_kernel<B, RPW, U>;
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)P.ctas, P.wk * P.wr * 32, (size_t)L.total, stream>>>(
      w.codes, w.n, w.k, w.lut, w.scales, w.rps, x, ldx, y, ldy,
      (int)L.lut_off, (int)L.red_off, P.wk, P.rows_max);
  return cudaGetLastError();
}

constexpr int64_t kMaxSmem = 227 * 1024;

int sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

}  // namespace

bool gemv_b_rows_supported(const WeightsView &w, int64_t batch) {
  if (w.format != TQ_FMT_B || batch < 1 || batch > 2) return false;
  if (w.k >= (int64_t)1 << 30) return false;
  const RowsPlan P = plan_rows<4>(w.n, w.k, sm_count());
  const int64_t red = (int64_t)P.wk * P.rows_max * batch * 4;
  const RowsLayout L = batch == 1 ? rows_layout<1, 8>(w.k, red)
                                  : rows_layout<2, 8>(w.k, red);
  return L.total <= kMaxSmem;
}

cudaError_t gemv_b_rows(const WeightsView &w, const __nv_bfloat16 *x,
                        int64_t batch, int64_t ldx, float *y, int64_t ldy,
                        cudaStream_t stream) {
  // 4 rows x 8 k-parts per warp: 128 contiguous bytes per row and step.
  const int sms = sm_count();
  if (batch == 1) return launch_rows<1, 4>(w, x, ldx, y, ldy, sms, stream);
  return launch_rows<2, 4>(w, x, ldx, y, ldy, sms, stream);
}

}  // namespace tq
