// Fused packed GEMM on the fifth-generation tensor cores (tcgen05), for the
// batches the GEMV kernels do not take (Format B batch >= 5, Format A
// batch >= 2), where x * W_hat^T becomes a real contraction:
//   Format A: y[b][n] = sum_p sum_g s_p[n][g] sum_{j in g} t_p[n][j] x[b][j]
//             (precisit.com page, "Three values and a shared scale"; second
//             plane per the FUCINA README, "The method")
//   Format B: y[b][n] = rho[n / rps] * sum_k LUT[code[n][k]] x[b][k]
//             (alphaneural.io page, sections 3.2, 3.3 and 4.2)
//
// One CTA computes a 128-row tile of y^T over the whole of K (or a cluster
// slice of it) for N = batch rounded up to 16 (<= 64), accumulating in tensor
// memory (128 lanes x N fp32 columns). Per 64-wide K block (and per plane):
//   - 16 decoder warps (four per TMEM lane quarter; a thread owns one row
//     and 16 k of the block) turn the codes of their rows into bf16 operands
//     and write them straight into tensor memory with tcgen05.st: the A
//     operand never passes through shared memory, whose bandwidth then only
//     carries the code-book lookups. Each weight w is split into
//     w_hi = bf16(w) and w_lo = bf16(w - w_hi): two MMAs (hi, then lo) give
//     products exact to ~2^-16 relative, well inside the 2e-3 tolerance, with
//     bf16 x used as is. For Format A, s*t splits exactly (an fp16 scale has
//     11 significant bits: 8 in s_hi, 3 in s_lo). The x tile is staged in
//     shared memory (operand B, K-major canonical layout). x and Format B
//     codes arrive through per-thread cp.async rings; Format A codes and
//     scales arrive in coalesced windows of 8 blocks that all decoders fetch
//     together (completion and reuse on mbarriers).
//   - One thread issues the 2 x 4 MMAs (M=128, N, K=16; A from tensor
//     memory, B from shared memory) of the block and commits them to the
//     stage's mbarrier, which frees the stage for the decoders. Tensor memory
//     holds the accumulator and 6 A stages of 64 columns (32 hi + 32 lo).
//   - After the last block the accumulator is read back with tcgen05.ld,
//     rho applied (Format B) and y stored.
// Waits are bounded; on a time-out the CTA writes NaN to its outputs, gives
// in-flight MMAs a bounded chance to finish, frees its tensor memory and
// exits. Decisions in front of warp-wide tcgen05 instructions are uniform.
#include <cooperative_groups.h>

#include "tq_common.cuh"
#include "tq_linear.cuh"
#include "tq_sm100_async.cuh"
#include "tq_sm100_mma.cuh"

namespace tq {
namespace {

constexpr int kTileM = 128;
constexpr int kMaxN = 64;
constexpr int kBlockK = 64;                       // k per stage
// Decoder warps per CTA (a multiple of 4: the TMEM lane quarters): 16, four
// per scheduler, 16 k per thread. The decode is bound by instruction issue
// and latency, so every warp the register budget allows is a decoder.
template <int FMT>
struct TcCfg {
  static constexpr int kDecoderWarps = 16;
  static constexpr int kKParts = kDecoderWarps / 4;  // k parts of a block
  static constexpr int kKPT = kBlockK / kKParts;     // k per decoder thread

  static constexpr int kXPerThread =
      (kMaxN * 8 + kDecoderWarps * 32 - 1) / (kDecoderWarps * 32);
  static constexpr int kThreads = 32 * (1 + kDecoderWarps);
};
constexpr int kStages = 6;                        // A in TMEM, x in smem
constexpr int kCodeDepth = 6;                     // x (and B code) ring depth
// Format A codes arrive in windows of kWinBlocks k-blocks: per row the
// window's 8 groups (104 code bytes) and 8 scales (16 bytes), fetched as
// 16-byte aligned chunks (so up to 128 + 32 bytes with the alignment slack)
// by all decoder threads together, lanes on consecutive chunks of a row.
constexpr int kWinBlocks = 8;
constexpr int kWinSlots = 3;                      // windows in the ring
constexpr int kWinRowCodes = 128;
constexpr int kWinRowBytes = kWinRowCodes + 32;
constexpr int kWinChunks = kTileM * kWinRowBytes / 16;  // 16-byte copies
constexpr uint32_t kTmemCols = 512;               // the whole tensor memory
constexpr uint32_t kAccCols = 64;                 // accumulator: N <= 64
constexpr uint32_t kStageCols = 64;               // A stage: 32 hi + 32 lo
constexpr int kLutStride = 128;                   // 32 lane copies x 4 B
constexpr int kLutBytes = 256 * kLutStride;       // 32 KB

// Offset of element (row r, k in [0,64)) inside an A (or x) K-block tile:
// four k16 sub-tiles of rows*32 bytes, each in the canonical K-major layout
// (LBO = 128: the second 8-k column; SBO = 256: the next 8 rows).
__device__ __forceinline__ uint32_t tile_off(int r, int k, int rows) {
  return (uint32_t)((k >> 4) * rows * 32 + (r >> 3) * 256 +
                    ((k >> 3) & 1) * 128 + (r & 7) * 16 + (k & 7) * 2);
}

struct TcParams {
  int ks_count;     // CTAs per cluster, each taking a slice of K
  int n_pad;        // N of the MMA (batch rounded up to 16)
  int stage_bytes;  // x tile
  int x_off;        // x tile offset inside a stage
  int ring_off, lut_off, bar_off, tmem_slot_off;
  int code_off, code_slot;  // B: kCodeDepth slots of 128 rows x 64 B;
                            // A: kWinSlots windows of 128 rows x 160 B
  int xring_off;            // x ring: kCodeDepth slots of n_pad rows x 128 B
  size_t smem;
};

// Asynchronous global -> shared copies; `n` < size bytes are read, the rest
// of the destination is zero-filled.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, int n) {
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

// Arrives on `bar` once every cp.async this thread issued so far has landed
// (the barrier's count includes this arrival).
__device__ __forceinline__ void cp_async_mbar_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar)
               : "memory");
}

// Warp-wide store of N (8 or 16) consecutive TMEM columns.
template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t ta,
                                             const uint32_t (&v)[N]) {
  if constexpr (N == 16) {
    tmem_st16(ta, v);
  } else {
    static_assert(N == 8, "8 or 16 columns");
    tmem_st8(ta, v);
  }
}

__device__ __forceinline__ uint32_t bf16_bits_rn(float v) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// Format B: 8 codes (two words) of one row -> 4 hi and 4 lo bf16 pairs. The
// table word of code c for this lane holds bf16(w) | bf16(w - bf16(w)) << 16.
__device__ __forceinline__ void decode8_b(uint32_t w0, uint32_t w1,
                                          uint32_t lut_base, uint32_t lane8,
                                          uint32_t (&hi)[4],
                                          uint32_t (&lo)[4]) {
  uint32_t v[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const uint32_t w = e < 4 ? w0 : w1;
    const uint32_t a2 = __byte_perm(w, lane8, 0x5504u | ((uint32_t)(e & 3) << 4));
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v[e]) : "r"(lut_base + (a2 >> 1)));
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    hi[q] = __byte_perm(v[2 * q], v[2 * q + 1], 0x5410u);
    lo[q] = __byte_perm(v[2 * q], v[2 * q + 1], 0x7632u);
  }
}

// Format A: trits 8c..8c+7 of the thread's 16, given as 2-bit fields
// (bit 2j: t_j != 0, bit 2j+1: t_j < 0) -> 4 hi and 4 lo pairs of s*t.
// s2 = s | s << 16 (hi or lo part of the scale in both halves); pair_tab[f]
// holds, for the 4 bits f of a pair, the keep mask (0xFFFF per nonzero half)
// and the sign mask (0x8000 per negative half), so a pair is one
// (s2 & keep) ^ sign. XOR (not OR) keeps a negative lo part exact.
__device__ __forceinline__ void decode8_a(uint32_t bits, int c,
                                          uint32_t s_hi2, uint32_t s_lo2,
                                          uint32_t pair_tab,
                                          uint32_t (&hi)[4],
                                          uint32_t (&lo)[4]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t f = (bits >> (16 * c + 4 * q)) & 15u;
    uint32_t keep, sign;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];"
                 : "=r"(keep), "=r"(sign)
                 : "r"(pair_tab + f * 8u));
    hi[q] = (s_hi2 & keep) ^ sign;
    lo[q] = (s_lo2 & keep) ^ sign;
  }
}

template <int FMT>
__global__ void __launch_bounds__(TcCfg<FMT>::kThreads, 1)
    gemm_tc_kernel(WeightsView w, const __nv_bfloat16 *__restrict__ x,
                   int64_t batch, int64_t ldx, float *__restrict__ y,
                   int64_t ldy, TcParams P) {
  constexpr int kDecoderWarps = TcCfg<FMT>::kDecoderWarps;
  constexpr int kKPT = TcCfg<FMT>::kKPT;
  constexpr int kXPerThread = TcCfg<FMT>::kXPerThread;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const uint32_t ring = sbase + P.ring_off;
  const uint32_t full0 = sbase + P.bar_off;           // full[s]: decoders done
  const uint32_t empty0 = full0 + 8 * kStages;        // empty[s]: MMAs done
  const uint32_t acc_bar = empty0 + 8 * kStages;      // accumulator ready
  const uint32_t wfull0 = acc_bar + 8;                // A window landed
  const uint32_t wempty0 = wfull0 + 8 * kWinSlots;    // A window consumed
  volatile uint32_t &tmem_slot =
      *reinterpret_cast<uint32_t *>(smem + P.tmem_slot_off);
  volatile int &abort_flag =
      *reinterpret_cast<int *>(smem + P.tmem_slot_off + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ks = blockIdx.x % P.ks_count;  // rank in the cluster
  const int64_t row0 = (int64_t)(blockIdx.x / P.ks_count) * kTileM;
  const int N = P.n_pad;
  const int64_t K = w.k;
  const int kblocks = (int)((K + kBlockK - 1) / kBlockK);
  const int planes = FMT == TQ_FMT_A ? w.planes : 1;
  const int iters_all = planes * kblocks;
  // this CTA's slice of the (plane, k-block) iterations
  const int it_begin = (int)((int64_t)iters_all * ks / P.ks_count);
  const int iters = (int)((int64_t)iters_all * (ks + 1) / P.ks_count) - it_begin;
  const uint32_t idesc = idesc_bf16_f32(kTileM, N);

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full0 + 8 * s, kDecoderWarps);
      mbar_init(empty0 + 8 * s, 1);
    }
    mbar_init(acc_bar, 1);
    if constexpr (FMT == TQ_FMT_A) {
      for (int s = 0; s < kWinSlots; ++s) {
        mbar_init(wfull0 + 8 * s, kDecoderWarps * 32);
        mbar_init(wempty0 + 8 * s, kDecoderWarps * 32);
      }
    }
    mbar_init_fence();
  }
  if (warp == 0) tmem_alloc(sbase + P.tmem_slot_off, kTmemCols);
  // Lookup tables.
  if constexpr (FMT == TQ_FMT_B) {
    // entry e, lane copy l at e*128 + 4*l: bf16(w) | bf16(w - bf16(w)) << 16
    for (int e = threadIdx.x; e < 256; e += blockDim.x) {
      const float v = __ldg(w.lut + e);
      const uint32_t h = bf16_bits_rn(v);
      const float hv = __uint_as_float(h << 16);
      const uint32_t l = bf16_bits_rn(v - hv);
      const uint32_t word = h | (l << 16);
      const uint4 w4 = make_uint4(word, word, word, word);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int jj = (j + e) & 7;
        *reinterpret_cast<uint4 *>(smem + P.lut_off + e * kLutStride + jj * 16) =
            w4;
      }
    }
  } else {
    // byte -> its 5 trits (least significant digit first) as 2-bit fields:
    // bit 2i: t_i != 0, bit 2i+1: t_i < 0
    uint16_t *tab = reinterpret_cast<uint16_t *>(smem + P.lut_off);
    for (int b = threadIdx.x; b < 256; b += blockDim.x) {
      uint32_t m = 0, rest = b < 243 ? b : 121;
#pragma unroll
      for (int i = 0; i < 5; ++i) {
        const uint32_t d = rest % 3;
        rest /= 3;
        if (d != 1) m |= 1u << (2 * i);
        if (d == 0) m |= 1u << (2 * i + 1);
      }
      tab[b] = (uint16_t)m;
    }
    // pair table (16 entries of keep, sign words) after the byte table,
    // indexed by two 2-bit fields
    uint32_t *ptab = reinterpret_cast<uint32_t *>(smem + P.lut_off + 512);
    for (int i = threadIdx.x; i < 16; i += blockDim.x) {
      const uint32_t z0 = i & 1, n0 = (i >> 1) & 1, z1 = (i >> 2) & 1,
                     n1 = (i >> 3) & 1;
      ptab[2 * i] = (z0 ? 0x0000FFFFu : 0u) | (z1 ? 0xFFFF0000u : 0u);
      ptab[2 * i + 1] = (z0 && n0 ? 0x00008000u : 0u) | (z1 && n1 ? 0x80000000u : 0u);
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = tmem_slot;

  if (warp == 0) {
    // ---- MMA issuer ----
    if (lane == 0) {
      int it = 0;
      for (; it < iters; ++it) {
        const int s = it % kStages;
        if (!mbar_wait(full0 + 8 * s, (it / kStages) & 1)) {
          abort_flag = 1;
          break;
        }
        tc_fence_after_sync();
        const uint32_t st = ring + s * P.stage_bytes;
        const uint32_t a_st = tmem + kAccCols + (uint32_t)s * kStageCols;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t bx =
              smem_desc_kmajor(st + P.x_off + ks * N * 32, 128, 256);
          // k16 step ks: 8 columns of the hi half, then of the lo half
          mma_bf16_ts(tmem, a_st + 8 * ks, bx, idesc,
                      (it > 0 || ks > 0) ? 1u : 0u);
          mma_bf16_ts(tmem, a_st + 32 + 8 * ks, bx, idesc, 1u);
        }
        mma_commit(empty0 + 8 * s);  // frees the stage when these finish
      }
      mma_commit(acc_bar);  // after every MMA issued above
    }
  } else {
    // ---- decoders ----
    const int wid = warp - 1;
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int kp = wid >> 2;       // which part of the 64 k of a block
    const int r = quarter * 32 + lane;
    const int64_t grow = row0 + r;
    const bool row_ok = grow < w.n;
    const uint32_t lane8 = (uint32_t)lane * 8u;
    const uint32_t lut_base = sbase + P.lut_off;
    const int64_t gpr = K / 64;  // Format A groups per row (G = 64)
    const int dt = wid * 32 + lane;  // decoder thread index
    // Format B codes stream into a per-thread ring of kCodeDepth blocks in
    // shared memory with cp.async (each thread reads back only the bytes its
    // own copies wrote), so kCodeDepth - 1 blocks of every row are in flight.
    const uint32_t code_ring = sbase + P.code_off + r * 64 + kp * kKPT;
    // Format A: the 16 trits k in [16 kp, 16 kp + 16) of a group lie in its
    // code bytes m_lo .. m_lo + 3, from trit a_off of byte m_lo on
    const int m_lo = (kKPT * kp) / 5;
    const int a_off = kKPT * kp - 5 * m_lo;
    // x chunks (16 B: one row, 8 k) ride in per-block cp.async groups: chunk
    // id of a block lands at x_ring(slot) + 16 id, copied and read by one
    // thread; slot = the block's iteration mod kCodeDepth.
    auto x_ring = [&](int slot) {
      return sbase + P.xring_off + (uint32_t)slot * (uint32_t)(N * 128);
    };
    // this thread's x chunks: row n, k offset 8c inside a block
    const __nv_bfloat16 *x_src[kXPerThread];
    bool x_live[kXPerThread];
#pragma unroll
    for (int q = 0; q < kXPerThread; ++q) {
      const int id = dt + q * kDecoderWarps * 32;
      const int n = id >> 3, c = id & 7;
      x_live[q] = id < N * 8;
      x_src[q] = n < batch ? x + (int64_t)n * ldx + 8 * c : nullptr;
    }
    // The next block to issue: its iteration, k-block and ring slot, kept
    // as counters (blocks are issued in order).
    int nx_it = 0, nx_slot = 0;
    int nx_kb = kblocks > 0 ? it_begin % kblocks : 0;
    auto issue_next = [&]() {
      if (nx_it < iters) {
        const uint32_t xd = x_ring(nx_slot);
#pragma unroll
        for (int q = 0; q < kXPerThread; ++q) {
          if (x_live[q]) {
            const int id = dt + q * kDecoderWarps * 32;
            const int64_t kk = (int64_t)nx_kb * kBlockK + 8 * (id & 7);
            const bool ok = x_src[q] != nullptr && kk < K;
            cp_async16(xd + 16 * id, ok ? x_src[q] + (int64_t)nx_kb * kBlockK : x,
                       ok ? 16 : 0);
          }
        }
        if constexpr (FMT == TQ_FMT_B) {
          const uint32_t dst = code_ring + (uint32_t)nx_slot * P.code_slot;
          const int64_t kk = (int64_t)nx_kb * kBlockK + kKPT * kp;
          const uint8_t *p = w.codes + (row_ok ? grow : 0) * K + kk;
#pragma unroll
          for (int j = 0; j < kKPT / 16; ++j) {
            const bool ok = row_ok && kk + 16 * j < K;
            cp_async16(dst + 16 * j, ok ? p + 16 * j : w.codes, ok ? 16 : 0);
          }
        }
      }
      ++nx_it;
      nx_slot = nx_slot + 1 == kCodeDepth ? 0 : nx_slot + 1;
      nx_kb = nx_kb + 1 == kblocks ? 0 : nx_kb + 1;
    };
    // Format A windows: the CTA's iterations [g0, g1) split at the plane
    // boundary into at most two runs, each cut into windows of kWinBlocks.
    const int g0 = it_begin, g1 = it_begin + iters;
    const int run0_end =
        kblocks > 0 ? min(g1, (g0 / kblocks + 1) * kblocks) : g0;
    const int n_win0 = (run0_end - g0 + kWinBlocks - 1) / kWinBlocks;
    const int n_win = n_win0 + (g1 - run0_end + kWinBlocks - 1) / kWinBlocks;
    auto win_lo = [&](int j) {
      return j < n_win0 ? g0 + kWinBlocks * j : run0_end + kWinBlocks * (j - n_win0);
    };
    auto win_hi = [&](int j) {
      return min(win_lo(j) + kWinBlocks, j < n_win0 ? run0_end : g1);
    };
    const int64_t plane_bytes = w.n * gpr * 13;  // Format A code bytes per plane
    // Every decoder thread copies its share of window j's chunks (chunk i:
    // row i / 10, the row's code chunk i % 10 < 8 or scale chunk i % 10 - 8)
    // into slot j % kWinSlots, once all decoders finished the window that
    // used the slot before; the copies complete on wfull[slot]. Chunks stop
    // at the end of the plane's codes or scales.
    auto issue_win = [&](int j) -> bool {
      if (j >= n_win) return true;
      const int slot = j % kWinSlots;
      if (j >= kWinSlots &&
          !mbar_wait(wempty0 + 8 * slot, ((j / kWinSlots) - 1) & 1))
        return false;
      const int gs = win_lo(j);
      const int plane = gs / kblocks, kb0 = gs - plane * kblocks;
      const uint8_t *cbase = w.codes + plane * w.codes_plane_stride;
      const uint8_t *cend = cbase + plane_bytes;
      const uint16_t *sbase_p = w.scales + plane * w.scales_plane_stride;
      const uint8_t *send = reinterpret_cast<const uint8_t *>(sbase_p + w.n * gpr);
      const uint32_t wslot = sbase + P.code_off + (uint32_t)slot * P.code_slot;
      for (int i = dt; i < kWinChunks; i += kDecoderWarps * 32) {
        const int row = i / 10, ch = i - 10 * row;
        const int64_t gr = row0 + row;
        if (gr >= w.n) continue;
        const int64_t gi0 = gr * gpr + kb0;
        const bool is_scale = ch >= 8;
        const uint8_t *first = is_scale
            ? reinterpret_cast<const uint8_t *>(sbase_p + gi0)
            : cbase + gi0 * 13;
        const uint8_t *src = reinterpret_cast<const uint8_t *>(
                                 reinterpret_cast<uintptr_t>(first) & ~(uintptr_t)15) +
                             16 * (is_scale ? ch - 8 : ch);
        const int64_t left = (is_scale ? send : cend) - src;
        const int nb = left >= 16 ? 16 : (left > 0 ? (int)left : 0);
        cp_async16(wslot + (uint32_t)(row * kWinRowBytes + 16 * ch),
                   nb > 0 ? src : w.codes, nb);
      }
      cp_async_mbar_arrive(wfull0 + 8 * slot);
      return true;
    };
    bool ok0 = true;
    if constexpr (FMT == TQ_FMT_A) {
      for (int j = 0; j + 1 < kWinSlots; ++j) ok0 = ok0 && issue_win(j);
    }
#pragma unroll
    for (int q = 0; q < kCodeDepth - 1; ++q) {
      issue_next();
      cp_async_commit();
    }
    if (!__all_sync(0xFFFFFFFFu, ok0)) abort_flag = 1;
    int wj = 0;                                  // current Format A window
    int w_lo = n_win > 0 ? win_lo(0) : 0, w_hi = n_win > 0 ? win_hi(0) : 0;
    uint32_t w_row = 0, c_off0 = 0, s_off0 = 0;  // its row base and offsets
    int s = 0, cur = 0;    // stage of block it, its x / code ring slot
    uint32_t e_par = 1;    // parity of the stage's previous use (from round 1)
    // A block's TMEM stores complete while the next block decodes: its
    // tcgen05.wait::st and full-barrier arrive come one iteration later.
    int s_prev = 0;
    bool pending = false;  // the previous block still awaits its arrive
    auto arrive_prev = [&]() {
      tmem_st_wait();
      tc_fence_before_sync();  // A stores -> ordered before the arrive
      __syncwarp();
      if (lane == 0) mbar_arrive(full0 + 8 * s_prev);
      pending = false;
    };
    // Every decision before a warp-wide (.sync.aligned) instruction is made
    // uniform across the warp.
    for (int it = 0; it < iters && !__any_sync(0xFFFFFFFFu, abort_flag != 0);
         ++it) {
      const int g = it_begin + it;
      issue_next();  // block it + kCodeDepth - 1
      cp_async_commit();
      cp_async_wait<kCodeDepth - 1>();  // this block's x (and B codes) landed
      uint32_t bits = 0;  // Format A: the thread's 16 trits, 2 bits each
      uint32_t s_hi = 0, s_lo = 0;
      uint32_t cw[4];
      if constexpr (FMT == TQ_FMT_A) {
        if (g == w_lo) {  // first block of window wj
          bool ok = issue_win(wj + kWinSlots - 1);
          ok = ok && mbar_wait(wfull0 + 8 * (wj % kWinSlots), (wj / kWinSlots) & 1);
          if (!__all_sync(0xFFFFFFFFu, ok)) {
            abort_flag = 1;
            break;
          }
          const int plane = g / kblocks, kb0 = g - plane * kblocks;
          const int64_t gi0 = (row_ok ? grow : 0) * gpr + kb0;
          c_off0 = (uint32_t)(reinterpret_cast<uintptr_t>(
                                  w.codes + plane * w.codes_plane_stride + gi0 * 13) & 15);
          s_off0 = (uint32_t)(reinterpret_cast<uintptr_t>(
                                  w.scales + plane * w.scales_plane_stride + gi0) & 15);
          w_row = sbase + P.code_off + (uint32_t)(wj % kWinSlots) * P.code_slot +
                  (uint32_t)(r * kWinRowBytes);
        }
        if (row_ok) {
          const uint32_t off = c_off0 + 13u * (uint32_t)(g - w_lo) + (uint32_t)m_lo;
          uint32_t w0, w1;
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w0) : "r"(w_row + (off & ~3u)));
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w1) : "r"(w_row + (off & ~3u) + 4));
          const uint32_t word = __funnelshift_r(w0, w1, 8u * (off & 3u));
          const uint16_t *tab =
              reinterpret_cast<const uint16_t *>(smem + P.lut_off);
          const uint32_t t0 = tab[word & 0xFFu], t1 = tab[(word >> 8) & 0xFFu],
                         t2 = tab[(word >> 16) & 0xFFu], t3 = tab[word >> 24];
          const uint32_t lo32 = t0 | t1 << 10 | t2 << 20 | t3 << 30;
          bits = __funnelshift_r(lo32, t3 >> 2, 2u * (uint32_t)a_off);
          uint16_t sbits;
          asm volatile("ld.shared.u16 %0, [%1];"
                       : "=h"(sbits)
                       : "r"(w_row + kWinRowCodes + s_off0 + 2u * (uint32_t)(g - w_lo)));
          const float sf = __half2float(__ushort_as_half(sbits));
          s_hi = bf16_bits_rn(sf);
          s_lo = bf16_bits_rn(sf - __uint_as_float(s_hi << 16));
          s_hi |= s_hi << 16;  // both halves of a pair
          s_lo |= s_lo << 16;
        }
        if (g + 1 == w_hi) {  // this thread is done reading window wj
          mbar_arrive(wempty0 + 8 * (wj % kWinSlots));
          ++wj;
          if (wj < n_win) {
            w_lo = win_lo(wj);
            w_hi = win_hi(wj);
          }
        }
      } else {
        const uint32_t src = code_ring + (uint32_t)cur * P.code_slot;
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(cw[0]), "=r"(cw[1]), "=r"(cw[2]), "=r"(cw[3])
                     : "r"(src));
        if (!row_ok) {
#pragma unroll
          for (int q = 0; q < 4; ++q) cw[q] = 0x79797979u;  // weight 0
        }
      }
      // decode this thread's kKPT k of its row: kKPT/2 hi and lo bf16 pairs
      uint32_t hi[kKPT / 2], lo[kKPT / 2];
#pragma unroll
      for (int cc = 0; cc < kKPT / 8; ++cc) {
        uint32_t h4[4], l4[4];
        if constexpr (FMT == TQ_FMT_B)
          decode8_b(cw[2 * cc], cw[2 * cc + 1], lut_base, lane8, h4, l4);
        else
          decode8_a(bits, cc, s_hi, s_lo, lut_base + 512, h4, l4);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          hi[4 * cc + q] = h4[q];
          lo[4 * cc + q] = l4[q];
        }
      }
      if (pending) arrive_prev();
      if (it >= kStages) {
        const bool ok = mbar_wait(empty0 + 8 * s, e_par);
        if (!__all_sync(0xFFFFFFFFu, ok)) {
          abort_flag = 1;
          break;
        }
      }
      tc_fence_after_sync();  // the stage's MMAs are done reading it
      {
        const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) + kAccCols +
                            (uint32_t)s * kStageCols +
                            (uint32_t)(kKPT / 2) * (uint32_t)kp;
        tmem_st_cols(ta, hi);
        tmem_st_cols(ta + 32, lo);
      }
      uint8_t *st = smem + P.ring_off + s * P.stage_bytes;
      // x tile: N rows x 64 k, 16 bytes per chunk, from this thread's ring
      {
        const uint32_t xs = x_ring(cur);
#pragma unroll
        for (int q = 0; q < kXPerThread; ++q) {
          const int id = dt + q * kDecoderWarps * 32;
          if (id < N * 8) {
            uint4 v;
            asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(xs + 16 * id));
            *reinterpret_cast<uint4 *>(st + P.x_off +
                                       tile_off(id >> 3, 8 * (id & 7), N)) = v;
          }
        }
      }
      fence_async_shared();   // x tile -> async proxy (MMA operand B)
      s_prev = s;
      pending = true;
      if (++s == kStages) {
        s = 0;
        e_par ^= 1u;
      }
      cur = cur + 1 == kCodeDepth ? 0 : cur + 1;
    }
    if (pending) arrive_prev();
    cp_async_wait<0>();
    // ---- epilogue: warps of the first half read their TMEM lane quarter ----
    if (kp == 0) {
      const bool ok = iters == 0 || mbar_wait(acc_bar, 0);
      if (!ok) abort_flag = 1;
      tc_fence_after_sync();
      float scale = 1.0f;
      if constexpr (FMT == TQ_FMT_B) {
        if (row_ok && w.scales != nullptr)
          scale = __half2float(__ushort_as_half(w.scales[grow / w.rps]));
      }
      float *part = reinterpret_cast<float *>(smem + P.ring_off);  // [128][N]
      for (int cb = 0; cb < N / 16; ++cb) {
        uint32_t v[16];
        tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + cb * 16, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int b = cb * 16 + i;
          float val = iters == 0 ? 0.0f : __uint_as_float(v[i]);
          if (abort_flag) val = __int_as_float(0x7FC00000);
          if (P.ks_count > 1) {
            part[r * N + b] = val;  // summed across the cluster below
          } else if (row_ok && b < batch) {
            y[(int64_t)b * ldy + grow] = scale * val;
          }
        }
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (P.ks_count > 1) {
    // Sum the cluster's partial tiles through distributed shared memory in
    // rank order (deterministic); this CTA finishes its share of the rows.
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    const float *part = reinterpret_cast<const float *>(smem + P.ring_off);
    const int r_lo = kTileM * ks / P.ks_count;
    const int r_hi = kTileM * (ks + 1) / P.ks_count;
    for (int i = threadIdx.x; i < (r_hi - r_lo) * N; i += blockDim.x) {
      const int rr = r_lo + i / N, b = i % N;
      const int64_t gr = row0 + rr;
      if (gr >= w.n || b >= batch) continue;
      float sum = 0.0f;
      for (int q = 0; q < P.ks_count; ++q)
        sum += cluster.map_shared_rank(part, q)[rr * N + b];
      float scale = 1.0f;
      if constexpr (FMT == TQ_FMT_B) {
        if (w.scales != nullptr)
          scale = __half2float(__ushort_as_half(w.scales[gr / w.rps]));
      }
      y[(int64_t)b * ldy + gr] = scale * sum;
    }
    cluster.sync();  // no CTA leaves while others read its partials
  }
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

TcParams plan_tc(int fmt, int64_t batch) {
  TcParams P{};
  const int64_t b = batch < kMaxN ? batch : kMaxN;
  P.n_pad = (int)((b + 15) / 16 * 16);
  P.stage_bytes = P.n_pad * kBlockK * 2;
  P.x_off = 0;
  P.ring_off = 0;
  P.code_slot = kTileM * (fmt == TQ_FMT_A ? kWinRowBytes : 64);
  P.code_off = kStages * P.stage_bytes;
  P.xring_off = P.code_off + (fmt == TQ_FMT_A ? kWinSlots : kCodeDepth) * P.code_slot;
  P.lut_off = P.xring_off + kCodeDepth * P.n_pad * 128;
  const int table = fmt == TQ_FMT_B ? kLutBytes : 512 + 128;
  P.bar_off = P.lut_off + table;
  P.tmem_slot_off = P.bar_off + (2 * kStages + 1 + 2 * kWinSlots) * 8 + 8;
  P.smem = (size_t)P.tmem_slot_off + 16;
  // one CTA per SM: each allocates the whole tensor memory
  if (P.smem < 120 * 1024) P.smem = 120 * 1024;
  return P;
}

// Cluster size (K slices per tile): the one that best fills whole waves of
// one CTA per SM, preferring no split.
int pick_ks(int64_t tiles, int iters, int sms) {
  int best = 1;
  double best_eff = 0.0;
  for (int ks = 1; ks <= 8 && ks <= iters; ++ks) {
    const double ctas = (double)(tiles * ks);
    const double waves = ctas / sms;
    const double eff = waves / ceil(waves) - 0.02 * (ks - 1);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = ks;
    }
  }
  return best;
}

template <int FMT>
cudaError_t launch_tc(const WeightsView &w, const __nv_bfloat16 *x,
                      int64_t batch, int64_t ldx, float *y, int64_t ldy,
                      cudaStream_t stream) {
  TcParams P = plan_tc(FMT, batch);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = (w.n + kTileM - 1) / kTileM;
  const int kblocks = (int)((w.k + kBlockK - 1) / kBlockK);
  const int iters = (FMT == TQ_FMT_A ? w.planes : 1) * kblocks;
  P.ks_count = pick_ks(tiles, iters, sms);
  auto kern = gemm_tc_kernel<FMT>;
  if (P.smem > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_limit<gemm_tc_kernel<FMT>>(227 * 1024);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(tiles * P.ks_count), 1, 1);
  cfg.blockDim = dim3(TcCfg<FMT>::kThreads, 1, 1);
  cfg.dynamicSmemBytes = P.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)P.ks_count;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, w, x, batch, ldx, y, ldy, P);
}

}  // namespace

bool gemm_tc_supported(const WeightsView &w, int64_t batch) {
  if (batch < 1) return false;
  if (w.format == TQ_FMT_B) return true;
  return w.format == TQ_FMT_A && w.group == 64;
}

cudaError_t gemm_tc(const WeightsView &w, const __nv_bfloat16 *x,
                    int64_t batch, int64_t ldx, float *y, int64_t ldy,
                    cudaStream_t stream) {
  for (int64_t b0 = 0; b0 < batch; b0 += kMaxN) {
    const int64_t nb = batch - b0 < kMaxN ? batch - b0 : kMaxN;
    const cudaError_t e =
        w.format == TQ_FMT_B
            ? launch_tc<TQ_FMT_B>(w, x + b0 * ldx, nb, ldx, y + b0 * ldy, ldy,
                                  stream)
            : launch_tc<TQ_FMT_A>(w, x + b0 * ldx, nb, ldx, y + b0 * ldy, ldy,
                                  stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace tq
