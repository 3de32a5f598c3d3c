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
  int64_t lut_off;
  int64_t total;
};

template <int B, int KP>
RowsLayout rows_layout(int64_t k) {
  const int64_t step = 16 * KP;
  const int64_t kpad = (k + step - 1) / step * step;
  RowsLayout L;
  L.x_bytes = kpad * B * 4;
  const int64_t base = kReservedSmem;
  L.lut_off = ((base + L.x_bytes + 65535) / 65536) * 65536 - base;
  L.total = L.lut_off + kLutBytes;
  return L;
}

template <int B, int RPW, int U>
__global__ void __launch_bounds__(kThreads, 1)
    gemv_b_rows_kernel(const uint8_t *__restrict__ codes, int64_t n,
                       int64_t k, const float *__restrict__ lut,
                       const uint16_t *__restrict__ rho, int rps,
                       const __nv_bfloat16 *__restrict__ x, int64_t ldx,
                       float *__restrict__ y, int64_t ldy, int lut_off) {
  constexpr int KP = 32 / RPW;    // k-parts (lanes) per row
  constexpr int STEP = 16 * KP;   // k per warp step
  extern __shared__ __align__(16) uint8_t smem[];
  const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(smem);
  const uint32_t xs = sbase;                          // permuted fp32 x
  const uint32_t lut_addr = sbase + (uint32_t)lut_off;
  const int64_t nsteps = (k + STEP - 1) / STEP;

  // Start this warp's first code loads before staging x and the code book.
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int r = lane / KP, p = lane % KP;
  const int64_t row_lo = (int64_t)blockIdx.x * n / gridDim.x;
  const int rows = (int)((int64_t)(blockIdx.x + 1) * n / gridDim.x - row_lo);
  const int nblk = (rows + RPW - 1) / RPW;

  // Stage x: element k of batch b goes to float index
  //   ((s*4 + q) * KP + p) * 4 * B + b * 4 + i,  k = s*STEP + p*16 + q*4 + i
  // so a lane's 4 chunks of a step are 16-byte loads at stride KP*16*B bytes.
  float *xsp = reinterpret_cast<float *>(smem);
  for (int64_t kk = threadIdx.x; kk < nsteps * STEP; kk += blockDim.x) {
    const int64_t s = kk / STEP;
    const int rem = (int)(kk % STEP);
    const int pp = rem >> 4, q = (rem >> 2) & 3, i = rem & 3;
    const int64_t base = (((s * 4 + q) * KP + pp) * B) * 4 + i;
#pragma unroll
    for (int b = 0; b < B; ++b)
      xsp[base + b * 4] = kk < k ? __bfloat162float(x[b * ldx + kk]) : 0.0f;
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
  // table in bytes 2-3. `fix` restores the base when the page trick is off.
  const bool paged = (lut_addr & 0xFFFFu) == 0;
  const uint32_t perm_op = (paged ? (lut_addr & 0xFFFF0000u) : 0u) | (lane * 4u);
  const uint32_t fix = paged ? 0u : lut_addr;

  for (int blk = warp; blk < nblk; blk += nwarps) {
    const int row = blk * RPW + r;
    const bool row_ok = row < rows;
    const uint8_t *cp = codes + (row_lo + (row_ok ? row : 0)) * k + p * 16;
    auto load = [&](int64_t s, uint32_t (&c)[4]) {
      c[0] = c[1] = c[2] = c[3] = 0x79797979u;  // code 121: weight 0
      if (row_ok && s < nsteps && s * STEP + p * 16 < k) {
        const uint4 v = ld_stream16(cp + s * STEP);
        c[0] = v.x; c[1] = v.y; c[2] = v.z; c[3] = v.w;
      }
    };
    uint32_t c[U][4];
#pragma unroll
    for (int u = 0; u < U; ++u) load(u, c[u]);
    float acc[B];
#pragma unroll
    for (int b = 0; b < B; ++b) acc[b] = 0.0f;
    for (int64_t s0 = 0; s0 < nsteps; s0 += U) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t s = s0 + u;
        if (s < nsteps) {
          uint32_t cur[4] = {c[u][0], c[u][1], c[u][2], c[u][3]};
          load(s + U, c[u]);
          const uint32_t xa = xs + (uint32_t)(((s * 4) * KP + p) * B * 16);
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
              const float wv = lds_f32(a + fix);
#pragma unroll
              for (int b = 0; b < B; ++b) acc[b] = fmaf(wv, xv[b][e], acc[b]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int b = 0; b < B; ++b) {
#pragma unroll
      for (int o = KP / 2; o >= 1; o >>= 1)
        acc[b] += __shfl_xor_sync(0xFFFFFFFFu, acc[b], o);
    }
    if (p == 0 && row_ok) {
      const int64_t grow = row_lo + row;
      const float scale =
          rho ? __half2float(__ushort_as_half(rho[grow / rps])) : 1.0f;
#pragma unroll
      for (int b = 0; b < B; ++b) y[(int64_t)b * ldy + grow] = scale * acc[b];
    }
  }
}

template <int B, int RPW>
cudaError_t launch_rows(const WeightsView &w, const __nv_bfloat16 *x,
                        int64_t ldx, float *y, int64_t ldy,
                        cudaStream_t stream) {
  constexpr int KP = 32 / RPW;
  constexpr int U = 8;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t ctas = sms < w.n ? sms : w.n;
  const int64_t rows_max = (w.n + ctas - 1) / ctas;
  const int64_t blocks = (rows_max + RPW - 1) / RPW;
  const int warps = (int)(blocks < kThreads / 32 ? blocks : kThreads / 32);
  const RowsLayout L = rows_layout<B, KP>(w.k);
  auto kern = gemv_b_rows_kernel<B, RPW, U>;
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)ctas, warps * 32, (size_t)L.total, stream>>>(
      w.codes, w.n, w.k, w.lut, w.scales, w.rps, x, ldx, y, ldy,
      (int)L.lut_off);
  return cudaGetLastError();
}

constexpr int64_t kMaxSmem = 227 * 1024;

}  // namespace

bool gemv_b_rows_supported(const WeightsView &w, int64_t batch) {
  if (w.format != TQ_FMT_B || batch < 1 || batch > 2) return false;
  const RowsLayout L = batch == 1 ? rows_layout<1, 8>(w.k)
                                  : rows_layout<2, 8>(w.k);
  return L.total <= kMaxSmem;
}

cudaError_t gemv_b_rows(const WeightsView &w, const __nv_bfloat16 *x,
                        int64_t batch, int64_t ldx, float *y, int64_t ldy,
                        cudaStream_t stream) {
  // 4 rows x 8 k-parts per warp: 128 contiguous bytes per row and step.
  if (batch == 1) return launch_rows<1, 4>(w, x, ldx, y, ldy, stream);
  return launch_rows<2, 4>(w, x, ldx, y, ldy, stream);
}

}  // namespace tq
