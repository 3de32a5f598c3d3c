// Format B fused GEMV at batch 1 and 2, streamed by the TMA engine
// (alphaneural.io page, sections 3.2, 3.3 and 4.2):
//   y[b][n] = rho[n / rps] * sum_k LUT[code[n][k]] * x[b][k].
//
// Two limits decide this kernel: bytes in flight per SM (warps prefetching
// into registers cannot hold enough) and shared-memory bandwidth (128 B per
// clock per SM, which the per-lane code-book lookups already half use).
//   - One CTA per SM owns rows [i*n/P, (i+1)*n/P). Warp 0 (one elected lane)
//     streams them through a ring of S shared-memory stages with 1-D bulk
//     copies: a stage holds a quad of 4 rows x one segment of C <= 1 KB (4
//     copies completing on the stage's mbarrier as transaction bytes); small
//     stages keep both the stage count and the consumer count high.
//   - W = 8 consumer warps, W dividing S and S >= 3W: stage s is always
//     consumed by warp s mod W, so each mbarrier's phases are awaited in
//     order by one warp, and each warp has its next stages in flight while
//     it works on one.
//   - A consumer warp's lanes are 4 rows x 8 k-parts: per 128-byte step a
//     lane takes 16 codes of its row, looks them up in its own copy of the
//     code book (entry e of lane l at byte e*256 + 4*l: conflict-free; the
//     byte permute of the code word is the whole address when the table sits
//     at a 64 KB aligned shared address, else one add) and multiplies by x
//     held in shared memory as fp32. The 4 rows of a k-part read the same x
//     bytes (broadcast), so x costs a quarter of the lookups' bandwidth.
//   - Per stage the 8 k-parts of each row are reduced with 3 shuffles and one
//     partial per (row, segment) is stored; the segments of a row are summed
//     in order at the end (deterministic) and rho is applied to the sum.
//   - Every wait is bounded; on a time-out the CTA writes NaN to its outputs,
//     waits (bounded) for its copies in flight and exits.
#include "tq_common.cuh"
#include "tq_linear.cuh"
#include "tq_sm100_async.cuh"

namespace tq {
namespace {

constexpr int kLutBytes = 256 * 256;   // 256 entries x 32 lane copies x 4 B
constexpr int kReservedSmem = 1024;    // system shared memory below the CTA's
constexpr int kMaxConsumers = 16;
constexpr int kMaxStages = 32;
constexpr int kRows = 4;               // rows per stage
constexpr int kParts = 8;              // k-parts (lanes) per row
constexpr int kStep = 16 * kParts;     // codes per row per warp step (128)

__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint4 lds_u32x4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ float4 lds_f32x4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
  return v;
}

struct StreamParams {
  int seg_bytes;    // C: codes per row per stage
  int nseg;         // segments per row
  int row_pitch;    // bytes between the 4 rows of a stage
  int stage_pitch;  // bytes between ring stages
  int stages;       // S
  int consumers;    // W, divides S
  int x_off, part_off, bar_off, lut_off, ring_off;
  int paged;        // table placed at a 64 KB aligned shared address
  int rows_max;
  size_t smem;
};

// Dot of one row segment (this lane's k-part) with x.
template <int B, bool PAGED>
__device__ __forceinline__ void segment_dot(uint32_t rowbuf, int seg_bytes,
                                            int T0, int p, uint32_t xs,
                                            uint32_t perm_op, uint32_t fix,
                                            float (&acc)[B]) {
#pragma unroll 2
  for (int t = 0; t * kStep < seg_bytes; ++t) {
    const int off = t * kStep + p * 16;
    if (off < seg_bytes) {
      const uint4 cv = lds_u32x4(rowbuf + off);
      const uint32_t cw[4] = {cv.x, cv.y, cv.z, cv.w};
      // x chunk (T, q, part p) at byte ((T*4 + q)*8 + p)*16*B + b*16
      const uint32_t xa = xs + (uint32_t)(((T0 + t) * 4 * kParts + p) * B * 16);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float xv[B][4];
#pragma unroll
        for (int b = 0; b < B; ++b) {
          const float4 f = lds_f32x4(xa + (q * kParts * B + b) * 16);
          xv[b][0] = f.x; xv[b][1] = f.y; xv[b][2] = f.z; xv[b][3] = f.w;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t a =
              __byte_perm(cw[q], perm_op, 0x7604u | ((uint32_t)e << 4));
          const float wv = lds_f32(PAGED ? a : a + fix);
#pragma unroll
          for (int b = 0; b < B; ++b) acc[b] = fmaf(wv, xv[b][e], acc[b]);
        }
      }
    }
  }
}

template <int B>
__global__ void __launch_bounds__(32 * (1 + kMaxConsumers), 1)
    gemv_b_stream_kernel(const uint8_t *__restrict__ codes, int64_t n,
                         int64_t k, const float *__restrict__ lut,
                         const uint16_t *__restrict__ rho, int rps,
                         const __nv_bfloat16 *__restrict__ x, int64_t ldx,
                         float *__restrict__ y, int64_t ldy, StreamParams P) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const uint32_t xs = sbase + P.x_off;
  const uint32_t ring = sbase + P.ring_off;
  const uint32_t lut_addr = sbase + P.lut_off;
  const uint32_t full0 = sbase + P.bar_off;      // full[s]
  const uint32_t empty0 = full0 + 8 * P.stages;  // empty[s]
  float *part = reinterpret_cast<float *>(smem + P.part_off);
  // set by any thread whose bounded wait timed out
  volatile int &abort_flag =
      *reinterpret_cast<int *>(smem + P.bar_off + 16 * kMaxStages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row_lo = (int64_t)blockIdx.x * n / gridDim.x;
  const int rows = (int)((int64_t)(blockIdx.x + 1) * n / gridDim.x - row_lo);
  const int quads = (rows + kRows - 1) / kRows;
  const int nchunks = quads * P.nseg;
  const int C = P.seg_bytes;
  const uint8_t *span = codes + row_lo * k;

  // Issue stage j (row quad j / nseg, segment j % nseg) into ring slot s.
  auto issue = [&](int j, int s) {
    const int q = j / P.nseg, seg = j - q * P.nseg;
    const int r0 = q * kRows;
    const int nr = rows - r0 < kRows ? rows - r0 : kRows;
    const uint32_t bar = full0 + 8 * s;
    mbar_arrive_expect_tx(bar, (uint32_t)(nr * C));
    for (int r = 0; r < nr; ++r)
      bulk_g2s(ring + s * P.stage_pitch + r * P.row_pitch,
               span + (int64_t)(r0 + r) * k + (int64_t)seg * C, (uint32_t)C,
               bar);
  };

  // Barriers, then the first S stages right away (before any staging).
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < P.stages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    mbar_init_fence();
    for (int j = 0; j < P.stages && j < nchunks; ++j) issue(j, j);
  }

  // Stage x as fp32: element k = 128*T + 16*p + 4*q + i of batch b goes to
  // float index (((T*4 + q)*8 + p)*B + b)*4 + i. 8 elements per load.
  float *xsp = reinterpret_cast<float *>(smem + P.x_off);
  const int kpad = (int)((k + kStep - 1) / kStep) * kStep;
  for (int v = threadIdx.x; v < kpad / 8; v += blockDim.x) {
    const int kk = v * 8;
    const int T = kk >> 7, pp = (kk >> 4) & 7, q0 = (kk >> 2) & 3;
#pragma unroll
    for (int b = 0; b < B; ++b) {
      uint4 raw = make_uint4(0, 0, 0, 0);
      if (kk < k) raw = *reinterpret_cast<const uint4 *>(x + b * ldx + kk);
      const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float4 f;
        f.x = __uint_as_float(wd[2 * h] << 16);
        f.y = __uint_as_float(wd[2 * h] & 0xFFFF0000u);
        f.z = __uint_as_float(wd[2 * h + 1] << 16);
        f.w = __uint_as_float(wd[2 * h + 1] & 0xFFFF0000u);
        const int idx = ((((T * 4 + q0 + h) * kParts + pp) * B) + b) * 4;
        *reinterpret_cast<float4 *>(xsp + idx) = f;
      }
    }
  }
  // Code book, one copy per lane, conflict-free rotated 16-byte stores.
  for (int e = threadIdx.x; e < 256; e += blockDim.x) {
    const float v = __ldg(lut + e);
    const float4 v4 = make_float4(v, v, v, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int jj = (j + e) & 7;
      *reinterpret_cast<float4 *>(smem + P.lut_off + e * 256 + jj * 16) = v4;
    }
  }
  __syncthreads();

  if (warp == 0) {
    // Producer: refill each stage once its consumer has released it.
    if (lane == 0) {
      for (int j = P.stages; j < nchunks && !abort_flag; ++j) {
        const int s = j % P.stages;
        if (!mbar_wait(empty0 + 8 * s, ((j / P.stages) - 1) & 1)) {
          abort_flag = 1;
          break;
        }
        issue(j, s);
      }
    }
  } else {
    const int wc = warp - 1;  // consumer index; owns stages s = wc mod W
    const int r = lane / kParts, p = lane % kParts;
    const bool paged = P.paged && (lut_addr & 0xFFFFu) == 0;
    const uint32_t perm_op =
        (paged ? (lut_addr & 0xFFFF0000u) : 0u) | ((uint32_t)lane * 4u);
    for (int j = wc; j < nchunks; j += P.consumers) {
      const int s = j % P.stages;
      if (!mbar_wait(full0 + 8 * s, (j / P.stages) & 1)) {
        abort_flag = 1;
        break;
      }
      const int q = j / P.nseg, seg = j - q * P.nseg;
      const int row = q * kRows + r;
      float acc[B];
#pragma unroll
      for (int b = 0; b < B; ++b) acc[b] = 0.0f;
      if (row < rows) {
        const uint32_t rowbuf = ring + s * P.stage_pitch + r * P.row_pitch;
        const int T0 = seg * C / kStep;  // C % 128 == 0 when nseg > 1
        if (paged)
          segment_dot<B, true>(rowbuf, C, T0, p, xs, perm_op, 0u, acc);
        else
          segment_dot<B, false>(rowbuf, C, T0, p, xs, perm_op, lut_addr, acc);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * s);  // stage reads are done
#pragma unroll
      for (int b = 0; b < B; ++b) {
#pragma unroll
        for (int o = kParts / 2; o >= 1; o >>= 1)
          acc[b] += __shfl_xor_sync(0xFFFFFFFFu, acc[b], o);
        if (p == 0 && row < rows) part[(row * P.nseg + seg) * B + b] = acc[b];
      }
      if (abort_flag) break;
    }
  }
  __syncthreads();

  if (abort_flag) {
    // Give the copies still in flight (at most S stages) a bounded chance to
    // land before the CTA's shared memory is released; outputs are poisoned.
    if (threadIdx.x == 0) {
      const int last = nchunks < P.stages ? nchunks : P.stages;
      for (int j = nchunks - last; j < nchunks; ++j)
        (void)mbar_wait(full0 + 8 * (j % P.stages), (j / P.stages) & 1);
    }
    for (int i = threadIdx.x; i < rows * B; i += blockDim.x)
      y[(int64_t)(i % B) * ldy + row_lo + i / B] = __int_as_float(0x7FC00000);
    return;
  }
  for (int i = threadIdx.x; i < rows * B; i += blockDim.x) {
    const int rr = i / B, b = i % B;
    float sum = 0.0f;
    for (int sg = 0; sg < P.nseg; ++sg) sum += part[(rr * P.nseg + sg) * B + b];
    const int64_t grow = row_lo + rr;
    const float scale =
        rho ? __half2float(__ushort_as_half(rho[grow / rps])) : 1.0f;
    y[(int64_t)b * ldy + grow] = scale * sum;
  }
}

// Lay out shared memory for one shape; stages == 0 when it does not fit.
// Each of the 8 consumer warps owns S/8 >= 3 stages, so that while it works
// on one stage its next ones are already being filled.
StreamParams plan_stream(int64_t n, int64_t k, int B, int64_t ctas,
                         int max_smem) {
  constexpr int kConsumers = 8;
  constexpr int kMinStages = 3 * kConsumers;
  StreamParams P{};
  P.rows_max = (int)((n + ctas - 1) / ctas);
  const int64_t kpad = (k + kStep - 1) / kStep * kStep;
  const int64_t x_bytes = kpad * B * 4;
  P.x_off = 0;
  P.part_off = (int)x_bytes;
  const int64_t quads = (P.rows_max + kRows - 1) / kRows;
  // The largest segment C (dividing k; a multiple of 128 unless it is the
  // whole row) that still leaves room for kMinStages stages.
  for (int cmax = 2048; cmax >= kStep; cmax /= 2) {
    int nseg = 0;
    for (int s = 1; s <= 1024; ++s) {
      if (k % s) continue;
      const int64_t C = k / s;
      if (C > cmax) continue;
      if (s > 1 && C % kStep) continue;
      nseg = s;
      break;
    }
    if (nseg == 0) continue;
    const int seg = (int)(k / nseg);
    const int row_pitch = (seg + 127) / 128 * 128;
    const int stage_pitch = kRows * row_pitch;
    const int64_t part_bytes = quads * kRows * nseg * B * 4;
    const int bar_off = (int)((x_bytes + part_bytes + 15) / 16 * 16);
    const int64_t front = (bar_off + 16 * kMaxStages + 16 + 255) / 256 * 256;
    int64_t lut_a = 65536 - kReservedSmem;  // 64 KB aligned shared address
    while (lut_a < front) lut_a += 65536;
    const int64_t st_a = (max_smem - (lut_a + kLutBytes)) / stage_pitch;
    const int64_t st_b = (max_smem - (front + kLutBytes)) / stage_pitch;
    const bool use_a = st_a >= kMinStages;
    int64_t st = use_a ? st_a : st_b;
    if (st > kMaxStages) st = kMaxStages;
    st = st / kConsumers * kConsumers;
    if (st < kMinStages) continue;
    P.nseg = nseg;
    P.seg_bytes = seg;
    P.row_pitch = row_pitch;
    P.stage_pitch = stage_pitch;
    P.bar_off = bar_off;
    P.paged = use_a ? 1 : 0;
    P.lut_off = (int)(use_a ? lut_a : front);
    P.ring_off = P.lut_off + kLutBytes;
    P.stages = (int)st;
    P.consumers = kConsumers;
    P.smem = (size_t)P.ring_off + (size_t)P.stages * P.stage_pitch;
    return P;
  }
  return P;
}

struct Device {
  int sms;
  int max_smem;
};

Device device_props() {
  Device d{148, 227 * 1024};
  int dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&d.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                         dev);
  return d;
}

template <int B>
cudaError_t launch_stream(const WeightsView &w, const __nv_bfloat16 *x,
                          int64_t ldx, float *y, int64_t ldy,
                          cudaStream_t stream) {
  const Device d = device_props();
  const int64_t ctas = d.sms < w.n ? d.sms : w.n;
  const StreamParams P = plan_stream(w.n, w.k, B, ctas, d.max_smem);
  auto kern = gemv_b_stream_kernel<B>;
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P.smem);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)ctas, 32 * (1 + P.consumers), P.smem, stream>>>(
      w.codes, w.n, w.k, w.lut, w.scales, w.rps, x, ldx, y, ldy, P);
  return cudaGetLastError();
}

}  // namespace

bool gemv_b_stream_supported(const WeightsView &w, int64_t batch) {
  if (w.format != TQ_FMT_B || batch < 1 || batch > 2) return false;
  if (w.k >= ((int64_t)1 << 24)) return false;
  const Device d = device_props();
  const int64_t ctas = d.sms < w.n ? d.sms : w.n;
  return plan_stream(w.n, w.k, (int)batch, ctas, d.max_smem).stages >= 2;
}

cudaError_t gemv_b_stream(const WeightsView &w, const __nv_bfloat16 *x,
                          int64_t batch, int64_t ldx, float *y, int64_t ldy,
                          cudaStream_t stream) {
  if (batch == 1) return launch_stream<1>(w, x, ldx, y, ldy, stream);
  return launch_stream<2>(w, x, ldx, y, ldy, stream);
}

}  // namespace tq
