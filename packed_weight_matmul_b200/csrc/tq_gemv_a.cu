// Format A fused GEMV at batch 1 (ternary-quantization page, sections on the
// group rule and the base-3 packing; the ternary-MoE page, two-plane
// reconstruction): y[n] = sum_p sum_g s_p[n,g] * sum_{j in g} t_p[n,j] x[j].
//
// Format A packs 4.3 weights into a byte, so at HBM speed an SM meets about
// 90 weights per clock: any per-weight decode step would be the bound. The
// kernel therefore never decodes a trit. A code byte m of a group holds the
// five trits of x positions 5m..5m+4, and the five-term sum over them can
// take only 243 values, one per byte value. For a window of 8 groups the
// CTA tabulates, for each of its 104 byte positions, all 243 partial sums
// ("activation tables", built once and reused by every row of the CTA);
// each code byte then costs one table load and one FMA with its group
// scale:
//   - Lane mapping: a warp walks rows; in step i (4 per window) lanes 0-12
//     take the 13 bytes of group 2i and lanes 13-25 those of group 2i+1, so
//     each lane reads one byte per step and its scale is the scale of one
//     group. Lanes 26-31 idle.
//   - The table of step i is [243][32] fp32 with lane l's entries in column
//     l: every lookup of a warp hits 32 distinct banks whatever the bytes.
//   - A cluster of KS CTAs splits the groups (K); each CTA holds its rows'
//     partial sums in shared memory, and rank q adds slice q of the rows over
//     the cluster's ranks in rank order (distributed shared memory): the
//     result does not depend on timing.
//   - Code bytes and scales are loaded a few rows ahead into registers and
//     prefetched into L2 further ahead.
#include <cooperative_groups.h>

#include <atomic>

#include "tq_common.cuh"
#include "tq_linear.cuh"

namespace tq {
namespace {

constexpr int kG = 64;                 // group size
constexpr int kNB = 13;                // bytes per group
constexpr int kWinGroups = 8;          // groups per table window
constexpr int kSteps = kWinGroups / 2;  // two groups per warp step
constexpr int kLanes = 2 * kNB;         // active lanes (26)
constexpr uint32_t kSub = 243u * 128u;  // one step's table: [243][32] fp32
// Bytes >= 243 read past the last table; the pad keeps them inside.
constexpr uint32_t kTabBytes = kSteps * kSub + 13u * 128u;
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kRing = 8;           // rows in registers ahead of use
constexpr int kL2Ahead = 32;       // rows prefetched into L2 ahead of use
constexpr int kSmemMax = 227 * 1024;

struct GemvAParams {
  int ks_count;      // CTAs per cluster (K slices)
  int rb_count;      // row blocks
  int rows_max;      // rows of the largest row block
  int planes_max;    // planes the partial-sum buffer holds
  int64_t ng;        // groups per row
};

__device__ __forceinline__ uint32_t ld_u8(const uint8_t *p) {
  uint32_t v;
  asm volatile("ld.global.nc.u8 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t ld_u16(const uint16_t *p) {
  uint32_t v;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ void prefetch_l2(const void *p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ float lds_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}

// Reduce 8 per-lane values across the warp: on return lane l holds, in
// v[0], the full sum of value index l >> 2.
__device__ __forceinline__ float butterfly8(float *v, int lane) {
  int m = 8;
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

__global__ void __launch_bounds__(kThreads, 1)
    gemv_a_kernel(WeightsView w, const __nv_bfloat16 *__restrict__ x,
                  float *__restrict__ y, GemvAParams P, ExpertsView E) {
  namespace cg = cooperative_groups;
  extern __shared__ __align__(16) uint8_t smem[];
  const uint32_t tab = (uint32_t)__cvta_generic_to_shared(smem);
  // [planes][rows_max] partial sums, then the CTA's x slice as fp32
  float *red = reinterpret_cast<float *>(smem + kTabBytes);
  float *xs_all = red + P.planes_max * P.rows_max;

  // Expert-indexed calls: token t = blockIdx.z multiplies x row t by the
  // matrix of expert ids[t] (plane 2 for the hot prefix e < n_hot) into y
  // row t. An id outside 0 .. n_experts - 1 computes on expert 0, reports
  // TQ_ERR_INVALID_ARG and leaves NaN in the row (every CTA of the cluster
  // reads the same id, so all take the same path).
  bool bad_id = false;
  if (E.ids != nullptr) {
    const int64_t t = blockIdx.z;
    int e = __ldg(E.ids + t);
    if (e < 0 || e >= E.n_experts) {
      bad_id = true;
      e = 0;
    }
    w.codes = E.codes + (int64_t)e * E.codes_stride;
    w.scales = E.scales + (int64_t)e * E.scales_stride;
    w.planes = e < E.n_hot ? 2 : 1;
    if (w.planes == 2) {
      // plane 2 lives in its own arrays: express it as an offset
      w.codes_plane_stride =
          (int64_t)(E.codes2 + (int64_t)e * E.codes_stride - w.codes);
      w.scales_plane_stride =
          (int64_t)(E.scales2 + (int64_t)e * E.scales_stride - w.scales);
    }
    x += t * E.ldx;
    y += t * E.ldy;
    if (bad_id && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0)
      report(E.status, TQ_ERR_INVALID_ARG);
  }

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ks = blockIdx.x;  // rank in the cluster = K slice
  const int rb = blockIdx.y;
  const int64_t row_lo = (int64_t)rb * w.n / P.rb_count;
  const int rows = (int)((int64_t)(rb + 1) * w.n / P.rb_count - row_lo);
  const int64_t g_lo = (int64_t)ks * P.ng / P.ks_count;
  const int64_t g_hi = (int64_t)(ks + 1) * P.ng / P.ks_count;

  // this warp's rows of the block
  const int r_lo = rows * warp / kWarps;
  const int r_n = rows * (warp + 1) / kWarps - r_lo;

  for (int i = threadIdx.x; i < P.planes_max * P.rows_max; i += kThreads)
    red[i] = 0.0f;
  // Clear the tables once: a byte >= 243 then reads a finite value (a
  // neighbouring table's entry or the pad).
  for (int i = threadIdx.x; i < (int)(kTabBytes / 16); i += kThreads)
    reinterpret_cast<float4 *>(smem)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  // x of the CTA's groups, once
  const int xn = (int)(g_hi - g_lo) * kG;
  for (int i = threadIdx.x; i < xn; i += kThreads)
    xs_all[i] = __bfloat162float(x[g_lo * kG + i]);

  // lane constant: which of the step's two groups the lane reads
  const int lg = lane >= kNB ? 1 : 0;
  const bool lane_on = lane < kLanes;
  const uint32_t lane_col = tab + 4u * (uint32_t)lane;
  const int64_t c_row = P.ng * kNB;  // bytes per row of codes

  for (int64_t w0 = g_lo; w0 < g_hi; w0 += kWinGroups) {
    const int gw = (int)(g_hi - w0 < kWinGroups ? g_hi - w0 : kWinGroups);
    __syncthreads();  // x is staged; the previous tables are no longer read
    // Build the tables: item (hi, p) fills the 9 entries v = 9*hi + lo of
    // byte position p (step p / 26, column p % 26).
    const int pos = kNB * gw;
    const float *xw = xs_all + (w0 - g_lo) * kG;
    for (int it = threadIdx.x; it < 27 * 128; it += kThreads) {
      const int hi = it >> 7, p = it & 127;
      if (p >= pos) continue;
      const int st = p / kLanes, col = p - st * kLanes;
      const int gl = 2 * st + (col >= kNB ? 1 : 0), q = col - (col >= kNB ? kNB : 0);
      const float *xp = xw + gl * kG + 5 * q;
      float xv[5];
#pragma unroll
      for (int j = 0; j < 5; ++j) xv[j] = (j < 4 || q < 12) ? xp[j] : 0.0f;
      const int d2 = hi % 3, d3 = (hi / 3) % 3, d4 = hi / 9;
      const float base = (float)(d2 - 1) * xv[2] + (float)(d3 - 1) * xv[3] +
                         (float)(d4 - 1) * xv[4];
      const uint32_t a = tab + (uint32_t)st * kSub + 4u * (uint32_t)col +
                         (uint32_t)(9 * hi) * 128u;
      const float m0 = -xv[0], p0 = xv[0];
#pragma unroll
      for (int d1 = 0; d1 < 3; ++d1) {
        const float b1 = base + (float)(d1 - 1) * xv[1];
        const uint32_t a1 = a + (uint32_t)(3 * d1) * 128u;
        asm volatile("st.shared.f32 [%0], %1;" ::"r"(a1), "f"(b1 + m0) : "memory");
        asm volatile("st.shared.f32 [%0], %1;" ::"r"(a1 + 128u), "f"(b1) : "memory");
        asm volatile("st.shared.f32 [%0], %1;" ::"r"(a1 + 256u), "f"(b1 + p0) : "memory");
      }
    }
    __syncthreads();

    // lane's steps that hold a byte of this window; the others load
    // nothing and read table column entries that are 0 (lanes 26-31) or
    // multiply by a scale of 0 (groups past the window).
    bool st_on[kSteps];
#pragma unroll
    for (int i = 0; i < kSteps; ++i) st_on[i] = lane_on && 2 * i + lg < gw;
    const bool sc_on = lane < gw;

    // In a full window every lane loads unconditionally: lanes 26-31 read
    // lane 0's byte (their table column is all zeros), lanes past the
    // window's groups read the last group's scale (never used).
    const bool full_win = gw == kWinGroups;
    const int loff = lane < kLanes ? lane : 0;
    const int soff = lane < gw ? lane : gw - 1;
    for (int pl = 0; pl < w.planes && r_n > 0; ++pl) {
      // this lane's code byte of step 0 and its scale, row r_lo
      const uint8_t *rb = w.codes + pl * w.codes_plane_stride +
                          ((row_lo + r_lo) * P.ng + w0) * kNB;
      const uint16_t *sb = w.scales + pl * w.scales_plane_stride +
                           (row_lo + r_lo) * P.ng + w0;
      const uint8_t *ldc = rb + (full_win ? loff : lane);
      const uint16_t *lds_ = sb + (full_win ? soff : lane);
      // the last row's pointers: rows past r_n reload it (values unused)
      const uint8_t *ldc_last = ldc + (int64_t)(r_n - 1) * c_row;
      const uint16_t *lds_last = lds_ + (int64_t)(r_n - 1) * P.ng;
      // all lanes prefetch: lane 1 the line of the window's last byte, the
      // others its first line (same address: one request), and the scales
      const uint8_t *pfc = rb + (lane == 1 ? kNB * gw - 1 : 0);
      const uint16_t *pfs = sb;
      int pf_r = 0;
      for (; pf_r < kL2Ahead && pf_r < r_n; ++pf_r) {
        prefetch_l2(pfc);
        prefetch_l2(pfs);
        pfc += c_row;
        pfs += P.ng;
      }
      uint32_t vb[kRing][kSteps];  // code bytes of the ring's rows
      uint32_t sr[kRing];          // raw fp16 scale (lanes 0..gw-1)
      auto load_row = [&](int d, bool ok) {
        if (full_win) {
          const uint8_t *c = ok ? ldc : ldc_last;
          const uint16_t *sp = ok ? lds_ : lds_last;
#pragma unroll
          for (int i = 0; i < kSteps; ++i) vb[d][i] = ld_u8(c + kLanes * i);
          sr[d] = ld_u16(sp);
        } else {
#pragma unroll
          for (int i = 0; i < kSteps; ++i)
            vb[d][i] = ok && st_on[i] ? ld_u8(ldc + kLanes * i) : 0u;
          sr[d] = ok && sc_on ? ld_u16(lds_) : 0u;
        }
        ldc += c_row;
        lds_ += P.ng;
      };
#pragma unroll
      for (int d = 0; d < kRing; ++d) load_row(d, d < r_n);
      for (int r0 = 0; r0 < r_n; r0 += kRing) {
        float v[kRing];
#pragma unroll
        for (int d = 0; d < kRing; ++d) {
          const float sf = __half2float(__ushort_as_half((uint16_t)sr[d]));
          float acc = 0.0f;
#pragma unroll
          for (int i = 0; i < kSteps; ++i) {
            const float sc = __shfl_sync(0xFFFFFFFFu, sf, 2 * i + lg);
            acc = fmaf(lds_f32(lane_col + (uint32_t)i * kSub + vb[d][i] * 128u),
                       sc, acc);
          }
          v[d] = acc;  // rows past r_n compute on zeros; not stored
          // refill the slot with row r0 + d + kRing
          load_row(d, r0 + d + kRing < r_n);
          if (pf_r < r_n) {
            prefetch_l2(pfc);
            prefetch_l2(pfs);
          }
          ++pf_r;
          pfc += c_row;
          pfs += P.ng;
        }
        // rows r0 .. r0+7: sum over the lanes, add into the plane's slot
        const float s = butterfly8(v, lane);
        const int idx = lane >> 2;
        if ((lane & 3) == 0 && r0 + idx < r_n)
          red[pl * P.rows_max + r_lo + r0 + idx] += s;
      }
    }
  }

  // Sum over the planes and the cluster's K slices, in rank order.
  cg::cluster_group cluster = cg::this_cluster();
  __syncthreads();
  cluster.sync();
  const int q_lo = rows * ks / P.ks_count, q_hi = rows * (ks + 1) / P.ks_count;
  for (int r = q_lo + (int)threadIdx.x; r < q_hi; r += kThreads) {
    float sum = 0.0f;
    for (int q = 0; q < P.ks_count; ++q) {
      const float *rr = cluster.map_shared_rank(red, q);
      for (int pl = 0; pl < w.planes; ++pl) sum += rr[pl * P.rows_max + r];
    }
    y[row_lo + r] = bad_id ? __int_as_float(0x7FC00000) : sum;
  }
  cluster.sync();  // no CTA leaves while others read its partial sums
}

}  // namespace

// Largest x slice (groups per CTA) staged in shared memory next to the tables.
constexpr int64_t kMaxSliceGroups = 96;

bool gemv_a_supported(const WeightsView &w, int64_t batch) {
  if (w.format != TQ_FMT_A || w.group != kG || batch != 1 || w.n < 1 ||
      w.k < kG)
    return false;
  const int64_t ng = w.k / kG;
  return (ng + 7) / 8 <= kMaxSliceGroups;  // slice of the 8-way split
}

namespace {

// Clusters of `ks` CTAs that can be resident at once (per device, cached:
// one CTA per SM whatever the request above the 114 KB half-SM mark).
int max_clusters(int dev, int ks, size_t smem) {
  static std::atomic<int> cache[16][4];
  const int slot = ks == 8 ? 3 : ks == 4 ? 2 : ks == 2 ? 1 : 0;
  if (dev >= 0 && dev < 16) {
    const int c = cache[dev][slot].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ks, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)ks;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // An error already pending belongs to the caller: leave it for them and
  // skip the query (the launcher then uses its SM-count fallback).
  if (cudaPeekAtLastError() != cudaSuccess) return 0;
  int n = 0;
  const cudaError_t q = cudaOccupancyMaxActiveClusters(&n, gemv_a_kernel, &cfg);
  if (q != cudaSuccess) {
    cudaGetLastError();  // clears only the query's own error
    return 0;
  }
  if (n < 1) return 0;
  if (dev >= 0 && dev < 16) cache[dev][slot].store(n, std::memory_order_relaxed);
  return n;
}

}  // namespace

namespace {

// One launch for `tokens` independent GEMVs (1 for a plain call): grid
// (K slices, row blocks, tokens), clusters along the K slices.
cudaError_t launch_gemv_a(const WeightsView &w, const __nv_bfloat16 *x,
                          float *y, const ExpertsView &E, int64_t tokens,
                          int planes_max, cudaStream_t stream) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (tokens < 1 || tokens > 65535) return cudaErrorInvalidValue;
  GemvAParams P;
  P.ng = w.k / kG;
  P.planes_max = planes_max;
  const size_t big = 160 * 1024;  // any request of one CTA per SM
  cudaError_t e = ensure_smem_limit<gemv_a_kernel>(kSmemMax);
  if (e != cudaSuccess) return e;
  // K slices: at most 8 (portable cluster), at least one full window each.
  // Each CTA owns an SM; its time is about windows x (its rows' lookups +
  // one table build). The resident clusters are shared by the tokens: take
  // the split with the least of (waves x that), waves counted over the
  // row blocks of every token.
  int best_ks = 1;
  int64_t best_rb = 1, best_ctas = 0;
  double best_cost = 0.0;
  for (int ks = 8; ks >= 1; ks /= 2) {
    if (ks > 1 && (P.ng + kWinGroups - 1) / kWinGroups < ks) continue;
    if ((P.ng + ks - 1) / ks > kMaxSliceGroups) break;
    int64_t res = max_clusters(dev, ks, big);
    if (res < 1) res = sms / ks;
    if (res < 1) res = 1;
    int64_t rb = res / tokens;
    if (rb < 1) rb = 1;
    if (rb > w.n) rb = w.n;
    const int64_t rows = (w.n + rb - 1) / rb;
    const int64_t waves = (rb * tokens + res - 1) / res;
    const int64_t wins = ((P.ng + ks - 1) / ks + kWinGroups - 1) / kWinGroups;
    const double cost =
        (double)waves * (double)wins *
        ((double)((rows + kWarps - 1) / kWarps) * planes_max * 40.0 + 300.0);
    if (best_ctas == 0 || cost < best_cost) {
      best_cost = cost;
      best_ctas = rb * ks;
      best_ks = ks;
      best_rb = rb;
    }
  }
  if (best_ctas == 0) return cudaErrorInvalidConfiguration;
  P.ks_count = best_ks;
  int64_t rb = best_rb;
  const int64_t slice = (P.ng + best_ks - 1) / best_ks;
  const int64_t fixed = (int64_t)kTabBytes + slice * kG * 4;
  // the partial sums must fit next to the tables and the x slice
  const int64_t red_cap = (kSmemMax - fixed) / (4 * planes_max);
  if ((w.n + rb - 1) / rb > red_cap) rb = (w.n + red_cap - 1) / red_cap;
  if (rb > 65535) return cudaErrorInvalidConfiguration;
  P.rb_count = (int)rb;
  P.rows_max = (int)((w.n + rb - 1) / rb);
  const size_t smem = (size_t)fixed + (size_t)planes_max * P.rows_max * 4;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)P.ks_count, (unsigned)P.rb_count,
                     (unsigned)tokens);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)P.ks_count;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_a_kernel, w, x, y, P, E);
}

}  // namespace

cudaError_t gemv_a(const WeightsView &w, const __nv_bfloat16 *x, float *y,
                   cudaStream_t stream) {
  ExpertsView E = {};
  return launch_gemv_a(w, x, y, E, 1, w.planes, stream);
}

cudaError_t gemv_a_experts(const WeightsView &w, const ExpertsView &E,
                           int64_t tokens, const __nv_bfloat16 *x, float *y,
                           cudaStream_t stream) {
  return launch_gemv_a(w, x, y, E, tokens, E.n_hot > 0 ? 2 : 1, stream);
}

}  // namespace tq
