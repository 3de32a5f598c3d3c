// Fused packed GEMM on the fifth-generation tensor cores (tcgen05), for the
// batches where x * W_hat^T is a real contraction:
//   Format A: y[b][n] = sum_p sum_g s_p[n][g] sum_{j in g} t_p[n][j] x[b][j]
//             (precisit.com page, "Three values and a shared scale"; second
//             plane per the FUCINA README, "The method")
//   Format B: y[b][n] = rho[n / rps] * sum_k LUT[code[n][k]] x[b][k]
//             (alphaneural.io page, sections 3.2, 3.3 and 4.2), also with
//             one code book per block of rows (section 8.3) and with 7-bit
//             indices into the layer's used words (section 8.1)
//
// Warp-specialised, one CTA per SM (it holds the whole tensor memory).
// Persistent clusters of `ks` CTAs walk the 128-row tiles of y^T: tile t,
// t + clusters, ...; with a split of K (ks > 1) each CTA of the cluster
// takes a slice of K of every tile. For each 128-wide k block ("iteration"):
//   - the code producer warp copies the tile's codes into a shared-memory
//     ring with tensor copies (TMA): Format B one 128-row x 128-code box
//     per block (7-bit indices: 128 rows x 112 bytes); Format A one box of codes and one of fp16 scales per window
//     of 4 blocks = 8 groups of 13 bytes, from the 16-byte boundary at or
//     below the window (when rows start on 16-byte boundaries; otherwise one
//     1-D bulk copy of each row's aligned run). Code boxes use the 128-byte
//     swizzle, so the decoders' row-wise reads spread over the banks. Few
//     large copies matter: the copy engine spends tens of cycles on each;
//   - the x producer copies the x tile (batch rounded up to 16 rows = N of
//     the MMA, 128 k) with two tensor copies of 64 k, 128-byte rows in the
//     K-major 128-byte-swizzle layout; rows past the batch and k past K read
//     as zero (boxes of 16-byte rows cost the copy engine about 20 cycles a
//     row, which made x the slowest input);
//   - 8 decoder warps (two per tensor-memory lane quarter; a thread owns one
//     row and 64 k) turn the codes into bf16 operands and store them straight
//     into tensor memory (tcgen05.st): A never passes through shared memory.
//     Each weight w is split into w_hi = bf16(w) and w_lo = bf16(w - w_hi),
//     so the two MMAs (hi, lo) carry 16 significant bits of w: exact for
//     Format A (an fp16 scale has 11), relative error <= 2^-17 for Format B.
//     A Format B book whose entries all lie on one integer grid takes one
//     exact operand, bf16(m), instead (see the set-up below);
//   - a waiter warp takes the waits for the x stage, the A stage and the
//     free accumulator and hands each ready stage to the MMA warp through a
//     named-barrier reduction, so the issuing thread only issues;
//   - one thread issues the 16 (or 8) MMAs (M = 128, N, K = 16, A from
//     tensor memory, B from shared memory) and commits them to the barriers
//     that free the x stage and the A stage, and after the tile's last block
//     to the accumulator barrier;
//   - 4 epilogue warps read the accumulator (double-buffered in tensor
//     memory, so the next tile's MMAs proceed meanwhile) and store y, or,
//     with a split, put the partial tile in shared memory; once every CTA
//     of the cluster has arrived on its "part full" barrier, each CTA adds
//     the `ks` partials of the rows it owns in rank order (distributed
//     shared memory; deterministic), applies rho and stores y, and arrives
//     on every CTA's "part free" barrier, which releases the buffers for
//     the next tile. This runs while the next tile's blocks stream in.
// Decoding uses a 64 KB table in shared memory at a 64 KB-aligned address,
// replicated once per lane, so that one byte permute of a code word with the
// lane's base word is the complete lookup address and a warp's lookups hit
// distinct banks:
//   Format B: entry c of lane l at tab + 256 c + 4 l holds bf16 hi | lo << 16
//             of LUT[c] (or bf16(m) on the grid); 7-bit indices use entries
//             0..127, the index moved to bits 8..14 of the lane's base word;
//             with a book per block of rows, each decoder warp keeps its
//             rows' book unreplicated (1 KB) instead;
//   Format A: entry b of lane l at tab + 256 b + 8 l holds, for the 5 trits
//             of code byte b, "selector bytes" 0x10 + 0x22 d (d = t + 1):
//             trits 0..3 in the first word, trits 2..4 in the second. Four
//             selector bytes, merged across code bytes with byte permutes,
//             select through one more byte permute the bf16 pair {-s, 0, +s}
//             of two weights (for the hi and for the lo part of the scale).
// All waits are bounded (normally 2 s); on a time-out the CTA stops, writes
// NaN to the outputs it owns, lets issued MMAs finish, frees its tensor
// memory and exits. Decisions in front of warp-wide tcgen05 instructions are
// uniform across the warp.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cooperative_groups.h>

#include <cstring>
#include <mutex>
#include <utility>

#include "tq_common.cuh"
#include "tq_linear.cuh"
#include "tq_sm100_async.cuh"
#include "tq_sm100_mma.cuh"

namespace tq {

// Test hooks (tq_testing_linear_wait_fault): a shorter wait limit and, when
// set, decoders that withhold their first "A stage ready" arrive.
std::atomic<uint64_t> g_test_wait_ns{0};
std::atomic<int> g_test_skip_first_arrive{0};
std::atomic<int> g_test_self_check{0};
// Mapped host buffer of the self-checking kernel's progress trace (or 0):
// entry [block * 8 + role] holds the last step the role reached.
std::atomic<unsigned long long> g_test_trace{0};
// Forced split of K and cluster cap (tq_testing_tc_split; 0 = automatic).
std::atomic<int> g_test_tc_ks{0};
std::atomic<int> g_test_tc_clusters{0};

// Record of the self-checking instantiation (test hook): [0] first
// violation (site << 48 | warp << 40 | block), [1] its value, [2] number of
// violations, [3] waits that gave up.
__device__ unsigned long long g_tc_check[4];

namespace {

constexpr int kTileM = 128;
constexpr int kMaxN = 64;
constexpr int kKB = 128;                 // k per iteration
constexpr int kAStages = 3;              // A stages in tensor memory
constexpr uint32_t kTmemCols = 512;      // the whole tensor memory
constexpr uint32_t kAccCols = 64;        // one accumulator (N <= 64)
constexpr uint32_t kAStage0 = 2 * kAccCols;
constexpr uint32_t kAStageCols = 128;    // 64 hi + 64 lo columns
constexpr int kDecWarps = 8;
constexpr int kWarpCodes = 0, kWarpX = 1, kWarpMma = 2, kWarpEpi = 3,
              kWarpDec = 7, kWarpWait = kWarpDec + kDecWarps;
constexpr int kThreads = 32 * (kWarpWait + 1);  // 512
constexpr int kBarIdStage = 1;  // named barrier: waiter -> MMA issuer
constexpr int kBarIdEpi = 2;    // named barrier: the 4 epilogue warps
// Decode variants of the decoder warps (Format A always takes kDecPair):
// Format B hi + lo table, single-operand table, table-free (entry c =
// u * (c - 121)), per-warp books (adaptive alphabet), 7-bit indices with a
// single-operand or a hi + lo table.
constexpr int kDecPair = 0, kDecGrid = 1, kDecIdent = 2, kDecAdaptive = 3,
              kDecB7Grid = 4, kDecB7Pair = 5;
constexpr int kMaxCodeStages = 8;
constexpr int kMaxXStages = 4;
constexpr uint32_t kBRow = 128;          // Format B row: 128 codes, swizzled
constexpr uint32_t kB7Row = 112;         // 7-bit alphabet row: 128 indices
constexpr int kAWin = 4;                 // Format A window: 4 blocks, 8 groups
constexpr uint32_t kARowCodes = 128;     // 104 code bytes + <= 15 skew
constexpr uint32_t kARow = 160;          // per-row copies: + 16 scale bytes
                                         // + <= 15 skew
constexpr uint32_t kAMapScales = kTileM * kARowCodes;  // tensor copies: the
constexpr uint32_t kAMapSRow = 32;       // scale rows (16 fp16) follow the codes
constexpr int kSmemMax = 227 * 1024;

// Barrier block (byte offsets).
constexpr uint32_t kBarCodeFull = 0, kBarCodeEmpty = 64, kBarXFull = 128,
                   kBarXEmpty = 160, kBarAFull = 192, kBarAEmpty = 216,
                   kBarAccFull = 240, kBarAccEmpty = 256, kBarDrain = 296,
                   kTmemSlot = 304, kAbort = 308, kUnit = 312,
                   kBarPartFull = 320, kBarPartFree = 328,
                   kBarBytes = 336;

struct TcPlan {
  int n_pad, ks, tiles, kblocks, iters;
  uint32_t base;  // window address where the dynamic shared memory starts
  uint32_t tab;   // 64 KB table, 64 KB aligned
  uint32_t code_lo, code_hi;   // code ring: stages [0, code_lo_n) at code_lo,
  int code_lo_n, code_stages;  // the others at code_hi
  uint32_t code_stage_bytes;
  uint32_t x_ring, x_stage_bytes;
  int x_stages;
  uint32_t red;  // partial tile [n_pad][128] fp32 (split of K only)
  uint32_t bars;
  int a_map;    // Format A windows by tensor copies (else one copy per row)
  uint64_t wait_ns;
  int skip_first_arrive;
  int grid_ok;  // Format B: the single-operand code-book path may be used
  size_t smem;
};

// Named-barrier reduction over `count` threads (whole warps): true when the
// predicate holds in every participating thread. No shared-memory access.
__device__ __forceinline__ bool bar_red_and(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n"
      " barrier.red.and.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t s) {
  return __byte_perm(a, b, s);
}

__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a)
               : "memory");
  return v;
}

// Table lookups: not volatile, so the compiler may schedule them freely; the
// table is complete before the barrier that precedes every role's loop.
__device__ __forceinline__ uint32_t lut32(uint32_t a) {
  uint32_t v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}

__device__ __forceinline__ uint2 lut64(uint32_t a) {
  uint2 v;
  asm("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}

__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y,
                                       uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(x),
               "r"(y), "r"(z), "r"(w)
               : "memory");
}

__device__ __forceinline__ uint32_t bf16_bits_rn(float v) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// End of the window that starts at iteration ws: at most `win` iterations,
// inside the slice and inside one plane.
__device__ __forceinline__ int window_end(int ws, int it1, int kblocks,
                                          int win) {
  const int plane_end = (ws / kblocks + 1) * kblocks;
  int we = ws + win;
  if (we > it1) we = it1;
  if (we > plane_end) we = plane_end;
  return we;
}

// Selector bytes 0x10 + 0x22 d of the five trits of code byte b (digits d,
// least significant first): trits 0..3 in .x, trits 2..4 in .y. A byte
// permute with selector byte 0x10 / 0x32 / 0x54 takes bytes 0-1 / 2-3 / 4-5
// of its two sources: -s / zero / +s.
__device__ __forceinline__ uint2 selector_entry(uint32_t b) {
  uint32_t rest = b < 243u ? b : 121u;  // invalid bytes: all trits 0
  uint32_t s[5];
#pragma unroll
  for (int i = 0; i < 5; ++i) {
    s[i] = 0x10u + 0x22u * (rest % 3u);
    rest /= 3u;
  }
  return make_uint2(s[0] | s[1] << 8 | s[2] << 16 | s[3] << 24,
                    s[2] | s[3] << 8 | s[4] << 16);
}

// Format B: 64 codes of one row (16 words) -> 32 hi and 32 lo bf16 pairs.
__device__ __forceinline__ void decode_b(const uint32_t (&cw)[16],
                                         uint32_t lane_tab, uint32_t (&hi)[32],
                                         uint32_t (&lo)[32]) {
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint32_t v0 = lut32(prmt(cw[j], lane_tab, 0x7604u));
    const uint32_t v1 = lut32(prmt(cw[j], lane_tab, 0x7614u));
    const uint32_t v2 = lut32(prmt(cw[j], lane_tab, 0x7624u));
    const uint32_t v3 = lut32(prmt(cw[j], lane_tab, 0x7634u));
    hi[2 * j] = prmt(v0, v1, 0x5410u);
    lo[2 * j] = prmt(v0, v1, 0x7632u);
    hi[2 * j + 1] = prmt(v2, v3, 0x5410u);
    lo[2 * j + 1] = prmt(v2, v3, 0x7632u);
  }
}

// Format B, single operand: 64 codes of one row -> 32 bf16 pairs.
__device__ __forceinline__ void decode_b_hi(const uint32_t (&cw)[16],
                                            uint32_t lane_tab,
                                            uint32_t (&hi)[32]) {
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint32_t v0 = lut32(prmt(cw[j], lane_tab, 0x7604u));
    const uint32_t v1 = lut32(prmt(cw[j], lane_tab, 0x7614u));
    const uint32_t v2 = lut32(prmt(cw[j], lane_tab, 0x7624u));
    const uint32_t v3 = lut32(prmt(cw[j], lane_tab, 0x7634u));
    hi[2 * j] = prmt(v0, v1, 0x5410u);
    hi[2 * j + 1] = prmt(v2, v3, 0x5410u);
  }
}

// bf16 pair of two fp32 values, `lo` in the low half.
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Format B, single operand, for a code book whose entry c is u * (c - 121),
// i.e. entry c = alpha * sum t_i a_i with code byte c = 121 + sum t_i 3^(i-1)
// and an ascending ternary ladder a_i = 3^(i-1) * a_1 (the least significant
// trit on the smallest step; the ladder 3^-(i-1) pairs it with the largest
// step and takes the table):
// 16 codes (one 16-byte load) -> 8 bf16 pairs of c - 121, without table
// lookups. A byte permute places code c in the low byte of the fp32 pattern
// of 2^23 + c, a packed fp32 subtraction of 2^23 + 121 leaves c - 121
// (exact), and one conversion packs two of them. Returns non-zero iff a code
// is >= 243 (invalid): per byte, bit 7 of (c & 0x7F) + 0x0D is set iff
// (c & 0x7F) >= 0x73, which with bit 7 of c set is c >= 0xF3.
__device__ __forceinline__ uint32_t decode_b_arith16(const uint4 v,
                                                     uint32_t (&hi)[8]) {
  const float2 bias = make_float2(-8388729.0f, -8388729.0f);  // -(2^23 + 121)
  const uint32_t cw[4] = {v.x, v.y, v.z, v.w};
  uint32_t bad = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t w = cw[j];
    float2 a = make_float2(__uint_as_float(prmt(w, 0x4B000000u, 0x7540u)),
                           __uint_as_float(prmt(w, 0x4B000000u, 0x7541u)));
    float2 b = make_float2(__uint_as_float(prmt(w, 0x4B000000u, 0x7542u)),
                           __uint_as_float(prmt(w, 0x4B000000u, 0x7543u)));
    a = __fadd2_rn(a, bias);
    b = __fadd2_rn(b, bias);
    hi[2 * j] = bf16x2_rn(a.x, a.y);
    hi[2 * j + 1] = bf16x2_rn(b.x, b.y);
    bad |= ((w & 0x7F7F7F7Fu) + 0x0D0D0D0Du) & w;
  }
  return bad & 0x80808080u;
}

// Format B with a code book per block of rows (adaptive alphabet): 64 codes
// of one row -> 32 hi and 32 lo bf16 pairs through the warp's compact book
// (256 words bf16 hi | lo << 16 at ctab).
__device__ __forceinline__ void decode_b_compact(const uint32_t (&cw)[16],
                                                 uint32_t ctab,
                                                 uint32_t (&hi)[32],
                                                 uint32_t (&lo)[32]) {
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint32_t v0 = lut32(ctab + ((cw[j] << 2) & 0x3FCu));
    const uint32_t v1 = lut32(ctab + ((cw[j] >> 6) & 0x3FCu));
    const uint32_t v2 = lut32(ctab + ((cw[j] >> 14) & 0x3FCu));
    const uint32_t v3 = lut32(ctab + ((cw[j] >> 22) & 0x3FCu));
    hi[2 * j] = prmt(v0, v1, 0x5410u);
    lo[2 * j] = prmt(v0, v1, 0x7632u);
    hi[2 * j + 1] = prmt(v2, v3, 0x5410u);
    lo[2 * j + 1] = prmt(v2, v3, 0x7632u);
  }
}

// 7-bit alphabet: table address of index J of a run of 64 7-bit indices
// (little-endian bit string d, index J at bits 7J .. 7J + 6). The index
// lands at bits 8..14, the entry pitch of the lane-replicated table.
template <int J>
__device__ __forceinline__ uint32_t b7_addr(const uint32_t (&d)[14],
                                            uint32_t lane_tab) {
  constexpr int bit = 7 * J, wd = bit >> 5, s = bit & 31;
  uint32_t v;
  if constexpr (s < 8)
    v = d[wd] << (8 - s);
  else if constexpr (s <= 25 || wd + 1 >= 14)
    v = d[wd] >> (s - 8);
  else
    v = __funnelshift_r(d[wd], d[wd + 1], s - 8);
  return (v & 0x7F00u) | lane_tab;
}

template <int J, bool LO>
__device__ __forceinline__ void decode_b7_pair(const uint32_t (&d)[14],
                                               uint32_t lane_tab,
                                               uint32_t (&hi)[32],
                                               uint32_t (&lo)[32]) {
  const uint32_t v0 = lut32(b7_addr<2 * J>(d, lane_tab));
  const uint32_t v1 = lut32(b7_addr<2 * J + 1>(d, lane_tab));
  hi[J] = prmt(v0, v1, 0x5410u);
  if constexpr (LO) lo[J] = prmt(v0, v1, 0x7632u);
}

template <bool LO, int... J>
__device__ __forceinline__ void decode_b7_all(const uint32_t (&d)[14],
                                              uint32_t lane_tab,
                                              uint32_t (&hi)[32],
                                              uint32_t (&lo)[32],
                                              std::integer_sequence<int, J...>) {
  (decode_b7_pair<J, LO>(d, lane_tab, hi, lo), ...);
}

// 7-bit alphabet: 64 indices of one row (56 bytes) -> 32 hi (and lo) bf16
// pairs through the lane-replicated table of the 128 used words.
template <bool LO>
__device__ __forceinline__ void decode_b7(const uint32_t (&d)[14],
                                          uint32_t lane_tab, uint32_t (&hi)[32],
                                          uint32_t (&lo)[32]) {
  decode_b7_all<LO>(d, lane_tab, hi, lo, std::make_integer_sequence<int, 32>{});
}

// Format A: one group (13 code bytes, realigned into b[0..3]) -> 32 hi and
// 32 lo bf16 pairs of s*t. (nh, ph) = (-s_hi with a zero upper half, +s_hi)
// are the byte sources of the selecting permute; (nl, pl) the same for s_lo.
__device__ __forceinline__ void decode_a(const uint32_t (&b)[4],
                                         uint32_t lane_tab, uint32_t nh,
                                         uint32_t ph, uint32_t nl, uint32_t pl,
                                         uint32_t (&hi)[32],
                                         uint32_t (&lo)[32]) {
  uint2 T[13];
#pragma unroll
  for (int m = 0; m < 13; ++m)
    T[m] = lut64(prmt(b[m >> 2], lane_tab, 0x7604u | ((uint32_t)(m & 3) << 4)));
  // E[j]: selector bytes of trits 4j .. 4j+3 (code byte m holds trits
  // 5m .. 5m+4); the pattern repeats every 4 code bytes (20 trits).
  uint32_t E[16];
#pragma unroll
  for (int p = 0; p < 3; ++p) {
    const uint2 t0 = T[4 * p], t1 = T[4 * p + 1], t2 = T[4 * p + 2],
                t3 = T[4 * p + 3];
    E[5 * p + 0] = t0.x;
    E[5 * p + 1] = prmt(t0.y, t1.x, 0x6542u);
    E[5 * p + 2] = prmt(t1.y, t2.x, 0x5421u);
    E[5 * p + 3] = prmt(t2.y, t3.x, 0x4210u);
    E[5 * p + 4] = prmt(t3.x, t3.y, 0x6321u);
  }
  E[15] = T[12].x;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint32_t e2 = E[j] >> 16;
    hi[2 * j] = prmt(nh, ph, E[j]);
    lo[2 * j] = prmt(nl, pl, E[j]);
    hi[2 * j + 1] = prmt(nh, ph, e2);
    lo[2 * j + 1] = prmt(nl, pl, e2);
  }
}

// Self-checking instantiation (CK): every address a role computes is checked
// against the region it must lie in; a violation is recorded (first one in
// full, all of them counted) and the access goes to a safe address instead.
__device__ __noinline__ void ck_record(uint32_t site, uint64_t value) {
  const unsigned long long tag =
      ((unsigned long long)site << 48) |
      ((unsigned long long)(threadIdx.x >> 5) << 40) | blockIdx.x;
  if (atomicCAS(&g_tc_check[0], 0ull, tag) == 0ull) g_tc_check[1] = value;
  atomicAdd(&g_tc_check[2], 1ull);
}

// This CTA's dynamic shared window [lo, lo + size) and a safe address in it.
struct SmemWin {
  uint32_t lo, size, safe;
};

template <bool CK>
__device__ __forceinline__ uint32_t ck_smem(const SmemWin &W, uint32_t a,
                                            uint32_t bytes, uint32_t site) {
  if constexpr (CK) {
    if (a < W.lo || a + bytes > W.lo + W.size ||
        (a & (bytes >= 16 ? 15u : bytes - 1u)) != 0u) {
      ck_record(site, a);
      return W.safe;  // in the window, aligned
    }
  }
  return a;
}

template <bool CK>
__device__ __forceinline__ uint32_t ck_tmem(uint32_t ta, uint32_t cols,
                                            uint32_t lane_base, uint32_t site) {
  if constexpr (CK) {
    if ((ta & 0xFFFFu) + cols > kTmemCols || (ta >> 16) != lane_base) {
      ck_record(site, ta);
      return (lane_base << 16) | kAStage0;
    }
  }
  return ta;
}

// Progress trace of the self-checking kernel: a store to mapped host memory
// (it outlives a fault of the context), made visible system-wide at once.
template <bool CK>
__device__ __forceinline__ void ck_trace(unsigned long long *trace, int role,
                                         int tile, int it, int step) {
  if constexpr (CK) {
    if (trace != nullptr) {
      const unsigned long long v = ((unsigned long long)(tile + 1) << 32) |
                                   ((unsigned long long)(it & 0xFFFF) << 16) |
                                   (unsigned long long)(step & 0xFFFF);
      asm volatile("st.volatile.global.u64 [%0], %1;" ::"l"(
                       trace + blockIdx.x * 8 + role),
                   "l"(v)
                   : "memory");
      __threadfence_system();
    }
  }
}

template <int FMT, bool CK>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const WeightsView w, int64_t batch, float *__restrict__ y,
                   int64_t ldy, const TcPlan P,
                   const __grid_constant__ CUtensorMap tmap_x,
                   const __grid_constant__ CUtensorMap tmap_c,
                   const __grid_constant__ CUtensorMap tmap_s,
                   unsigned long long *trace) {
  constexpr int kWin = FMT == TQ_FMT_A ? kAWin : 1;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t base = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ks = P.ks;
  const int nclusters = (int)gridDim.x / ks;
  const int cid = (int)blockIdx.x / ks;
  const int64_t N = w.n, K = w.k;
  const int n_pad = P.n_pad;
  const int nb = (int)(batch < n_pad ? batch : n_pad);
  const int64_t gpr = K / 64;  // Format A groups per row
  const int rank = ks > 1 ? (int)cluster_rank() : 0;
  // this CTA's iterations of every tile
  const int it0 = (int)((int64_t)P.iters * rank / ks);
  const int it1 = (int)((int64_t)P.iters * (rank + 1) / ks);
  // rows of every tile this CTA owns in the cluster reduction: whole groups
  // of 4 rows (one 16-byte vector of a partial-tile column)
  const int r_lo = 4 * (kTileM / 4 * rank / ks),
            r_hi = 4 * (kTileM / 4 * (rank + 1) / ks);
  // partial tile of a K split (same offset in every CTA of the cluster)
  float *const part = reinterpret_cast<float *>(smem + (P.red - P.base));

  // The plan places everything for a window at P.base. A CTA's own shared
  // addresses need not start there: in a cluster they also name the CTA's
  // rank (a shared::cta address is a shared::cluster one), so every planned
  // address moves by this CTA's offset. It keeps the table's 64 KB alignment
  // unless it is not a multiple of 64 KB: then no work is safe, the outputs
  // it owns are NaN, and a CTA of a cluster still takes the cluster's two
  // barriers (its peers wait for its partial tiles in vain, time out and
  // write NaN too).
  // The next kernel on the stream may be scheduled onto SMs this grid frees.
  pdl_launch_dependents();
  const uint32_t delta = base - P.base;
  if ((delta & 0xFFFFu) != 0u) {
    pdl_wait();
    const float qnan = __int_as_float(0x7FC00000);
    if (ks == 1) {
      for (int t = cid; t < P.tiles; t += nclusters)
        for (int i = threadIdx.x; i < kTileM * nb; i += blockDim.x) {
          const int64_t row = (int64_t)t * kTileM + i % kTileM;
          if (row < N) y[(int64_t)(i / kTileM) * ldy + row] = qnan;
        }
    } else {
      namespace cg = cooperative_groups;
      cg::cluster_group cluster = cg::this_cluster();
      cluster.sync();
      const int own = r_hi - r_lo;
      for (int t = cid; t < P.tiles; t += nclusters)
        for (int i = threadIdx.x; i < own * nb; i += blockDim.x) {
          const int64_t row = (int64_t)t * kTileM + r_lo + i % own;
          if (row < N) y[(int64_t)(i / own) * ldy + row] = qnan;
        }
      cluster.sync();
    }
    return;
  }
  const uint32_t tab = P.tab + delta;
  const uint32_t B0 = P.bars + delta;
  const uint32_t x_ring = P.x_ring + delta;
  const uint32_t code_lo = P.code_lo + delta, code_hi = P.code_hi + delta;
  const uint32_t abort_addr = B0 + kAbort;
  const uint64_t lim = P.wait_ns;
  const SmemWin W{base, (uint32_t)P.smem, B0};

  auto code_stage = [&](int s) -> uint32_t {
    return s < P.code_lo_n
               ? code_lo + (uint32_t)s * P.code_stage_bytes
               : code_hi + (uint32_t)(s - P.code_lo_n) * P.code_stage_bytes;
  };

  // ---- set-up -------------------------------------------------------------
  if (threadIdx.x == 0) {
    if constexpr (CK) {
      ck_smem<CK>(W, tab, 0x10000u, 1);
      ck_smem<CK>(W, B0, kBarBytes, 1);
      ck_smem<CK>(W, x_ring, (uint32_t)P.x_stages * P.x_stage_bytes, 1);
      if (P.ks > 1) ck_smem<CK>(W, P.red + delta, (uint32_t)(kTileM * P.n_pad * 4), 1);
      for (int s = 0; s < P.code_stages; ++s)
        ck_smem<CK>(W, code_stage(s), P.code_stage_bytes, 1);
    }
    st_volatile_s32(abort_addr, 0);
    for (int s = 0; s < P.code_stages; ++s) {
      mbar_init(B0 + kBarCodeFull + 8 * s, 1);
      mbar_init(B0 + kBarCodeEmpty + 8 * s, kDecWarps);
    }
    for (int s = 0; s < P.x_stages; ++s) {
      mbar_init(B0 + kBarXFull + 8 * s, 1);
      mbar_init(B0 + kBarXEmpty + 8 * s, 1);
    }
    for (int s = 0; s < kAStages; ++s) {
      mbar_init(B0 + kBarAFull + 8 * s, kDecWarps);
      mbar_init(B0 + kBarAEmpty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(B0 + kBarAccFull + 8 * b, 1);
      mbar_init(B0 + kBarAccEmpty + 8 * b, 4);
    }
    mbar_init(B0 + kBarDrain, 1);
    if (ks > 1) {
      mbar_init(B0 + kBarPartFull, (uint32_t)ks);
      mbar_init(B0 + kBarPartFree, (uint32_t)ks);
    }
    st_volatile_s32(B0 + kUnit, 0x7F800000);  // +inf
    mbar_init_fence();
  }
  if (warp == kWarpMma) {
    __syncwarp();
    tmem_alloc(B0 + kTmemSlot, kTmemCols);
  }
  if (warp == kWarpX && lane == 0)
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmap_x) : "memory");
  if (warp == kWarpCodes && lane == 0 && (FMT == TQ_FMT_B || P.a_map)) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmap_c) : "memory");
    if (FMT == TQ_FMT_A)
      asm volatile("prefetch.tensormap [%0];" ::"l"(&tmap_s) : "memory");
  }
  // While the kernel before this one on the stream finishes: warm L2 with
  // the code boxes of this CTA's first stages (Format B); then wait for that
  // kernel's completion before reading user memory (the code book first).
  if constexpr (FMT == TQ_FMT_B) {
    if (warp == kWarpCodes && lane == 0 && cid < P.tiles) {
      const bool b7p = w.format == TQ_FMT_B7;
      const int pre = it1 - it0 < P.code_stages ? it1 - it0 : P.code_stages;
      for (int i = 0; i < pre; ++i)
        tma_prefetch_2d(&tmap_c, (it0 + i) * (int)(b7p ? kB7Row : kKB),
                        cid * kTileM);
    }
  }
  pdl_wait();
  // Format B: when every code-book entry is an integer multiple m of one
  // unit u (|m| <= 256, to 2^-20 of the entry; e.g. the balanced-ternary
  // ladder 3^-(i-1), whose 243 words are the integers -121..121 in units of
  // alpha / 81), the operand is bf16(m), exact: one MMA per k step, and u
  // multiplies the accumulator in the epilogue. The representation error,
  // 2^-20, is below that of the hi + lo split (2^-17). Otherwise each entry
  // becomes bf16 hi + lo (two MMAs). u is the smallest non-zero |entry|; the
  // test runs in every CTA on the same table, so all CTAs agree.
  bool grid = false, ident = false;
  float unit = 1.0f;
  // adaptive alphabet: every decoder warp builds its rows' compact book per
  // tile in the table region; no shared table, no single-operand path
  const bool adaptive = FMT == TQ_FMT_B && w.lut_rows > 0;
  // 7-bit alphabet: 7-bit indices into a book of the 128 used words
  const bool b7 = FMT == TQ_FMT_B && w.format == TQ_FMT_B7;
  const int n_words = b7 ? 128 : 243;
  if (FMT == TQ_FMT_B && !adaptive) {
    __syncthreads();  // the unit word is initialised
    float lv = 0.0f;
    if ((int)threadIdx.x < n_words) {
      lv = __ldg(w.lut + threadIdx.x);
      const float a = fabsf(lv);
      if (a > 0.0f && a <= 3.4028235e38f)
        atom_min_shared_u32(B0 + kUnit, __float_as_uint(a));
    }
    __syncthreads();
    const float u = __int_as_float(ld_volatile_s32(B0 + kUnit));
    bool ok = true, id_ok = true;
    if ((int)threadIdx.x < n_words) {
      const float m = rintf(__fdiv_rn(lv, u));
      ok = u <= 3.4028235e38f && fabsf(m) <= 256.0f &&
           fabs((double)lv - (double)u * (double)m) <=
               ldexp(fabs((double)lv), -20);
      id_ok = m == (float)((int)threadIdx.x - 121);
    }
    grid = __syncthreads_and(ok) != 0 && P.grid_ok != 0;
    // m = c - 121 for every word (an ascending ternary ladder): decode
    // without the table
    const bool all_id = __syncthreads_and(id_ok) != 0;
    ident = grid && !b7 && all_id;
    if (grid) unit = u;
  }
  // the lane-replicated table
  if (FMT == TQ_FMT_B && !adaptive && !ident) {
    for (int i = threadIdx.x; i < 256 * 8; i += blockDim.x) {
      const int e = i >> 3, j = i & 7;
      // entries past the book (7-bit alphabet: 128 words) are never read
      const float v = !b7 || e < 128 ? __ldg(w.lut + e)
                                     : __int_as_float(0x7FC00000);
      uint32_t word;
      if (grid) {
        // bf16(m) in the low half; entries past the words stay NaN
        word = e < n_words ? bf16_bits_rn(rintf(__fdiv_rn(v, unit))) : 0x7FC0u;
      } else {
        const uint32_t h = bf16_bits_rn(v);
        const uint32_t l = bf16_bits_rn(v - __uint_as_float(h << 16));
        word = h | l << 16;
      }
      sts128(tab + (uint32_t)e * 256u + (uint32_t)j * 16u, word, word, word,
             word);
    }
  } else if (FMT == TQ_FMT_A) {
    for (int i = threadIdx.x; i < 256 * 16; i += blockDim.x) {
      const int e = i >> 4, j = i & 15;
      const uint2 v = selector_entry((uint32_t)e);
      sts128(tab + (uint32_t)e * 256u + (uint32_t)j * 16u, v.x, v.y, v.x,
             v.y);
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  // with a split of K, peers arrive on this CTA's partial-tile barriers:
  // every CTA of the cluster has initialised its barriers after this
  if (ks > 1) cooperative_groups::this_cluster().sync();
  tc_fence_after_sync();
  uint32_t tmem;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(tmem) : "r"(B0 + kTmemSlot)
               : "memory");

  if (warp == kWarpCodes) {
    // ---- code producer: each window's codes (and scales) ---------------------
    int s = 0, u = 0;  // ring slot, windows issued so far
    uint32_t ph = 0;   // (u / code_stages) & 1, kept without a division
    bool ok = true;
    for (int t = cid; ok && t < P.tiles; t += nclusters) {
      const int64_t row0 = (int64_t)t * kTileM;
      const int rows = (int)(N - row0 < kTileM ? N - row0 : kTileM);
      for (int ws = it0; ws < it1;) {
        const int we =
            FMT == TQ_FMT_B ? ws + 1 : window_end(ws, it1, P.kblocks, kWin);
        if (u >= P.code_stages)
          ok = mbar_wait(B0 + kBarCodeEmpty + 8 * s, ph ^ 1u, abort_addr, lim);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if constexpr (CK) if (!ok && lane == 0) ck_record(21, (uint64_t)u);
        if (!ok) break;
        const uint32_t full = B0 + kBarCodeFull + 8 * s;
        const uint32_t dst0 = code_stage(s);
        if (lane == 0) ck_trace<CK>(trace, 0, t, ws, 1);
        if constexpr (FMT == TQ_FMT_B) {
          // one box of 128 rows x 128 codes, 128-byte swizzle (16-byte chunk
          // c of row r lands at chunk c ^ (r & 7)); rows past N and codes
          // past K read as zero, and the decoders mask them. 7-bit alphabet:
          // 128 rows x 112 bytes (128 indices), not swizzled
          if (lane == 0) {
            const uint32_t bytes = kTileM * (b7 ? kB7Row : kBRow);
            uint32_t d = dst0;
            if constexpr (CK) d = ck_smem<CK>(W, d, bytes, 2);
            mbar_arrive_expect_tx(full, bytes);
            tma_load_2d(d, &tmap_c, ws * (b7 ? kB7Row : kKB), (int)row0, full);
          }
          __syncwarp();
        } else if (P.a_map) {
          // the window's 8 groups of every row: codes from the 16-byte
          // boundary at or below the first byte (128 bytes, 128-byte
          // swizzle), scales from the 8-scale boundary (16 fp16)
          const int plane = ws / P.kblocks;
          const int g0 = 2 * (ws - plane * P.kblocks);
          if (lane == 0) {
            uint32_t d = dst0;
            if constexpr (CK) d = ck_smem<CK>(W, d, P.code_stage_bytes, 4);
            mbar_arrive_expect_tx(full, kTileM * (kARowCodes + kAMapSRow));
            tma_load_3d(d, &tmap_c, (13 * g0) & ~15, (int)row0, plane, full);
            tma_load_3d(d + kAMapScales, &tmap_s, g0 & ~7, (int)row0, plane,
                        full);
          }
          __syncwarp();
        } else {
          const int plane = ws / P.kblocks;
          const int64_t g0 = 2 * (int64_t)(ws - plane * P.kblocks);
          const int64_t want = 2 * (int64_t)(we - ws);
          const uintptr_t ng = (uintptr_t)(want < gpr - g0 ? want : gpr - g0);
          const uintptr_t cbase = reinterpret_cast<uintptr_t>(w.codes) +
                                  (uintptr_t)(plane * w.codes_plane_stride);
          const uintptr_t sbase =
              reinterpret_cast<uintptr_t>(w.scales) +
              (uintptr_t)(2 * plane * w.scales_plane_stride);
          const uintptr_t m16 = ~(uintptr_t)15;
          uint32_t bytes = 0;
          for (int r = lane; r < rows; r += 32) {
            const int64_t gi = (row0 + r) * gpr + g0;
            const uintptr_t c = cbase + (uintptr_t)(gi * 13);
            const uintptr_t sc = sbase + (uintptr_t)(gi * 2);
            bytes += (uint32_t)(((c + 13 * ng + 15) & m16) - (c & m16));
            bytes += (uint32_t)(((sc + 2 * ng + 15) & m16) - (sc & m16));
          }
          bytes = __reduce_add_sync(0xFFFFFFFFu, bytes);
          if (lane == 0) mbar_arrive_expect_tx(full, bytes);
          __syncwarp();
          for (int r = lane; r < rows; r += 32) {
            const int64_t gi = (row0 + r) * gpr + g0;
            const uintptr_t c = cbase + (uintptr_t)(gi * 13);
            const uintptr_t sc = sbase + (uintptr_t)(gi * 2);
            uint32_t dst = dst0 + (uint32_t)r * kARow;
            const uint32_t csz = (uint32_t)(((c + 13 * ng + 15) & m16) - (c & m16));
            const uint32_t ssz = (uint32_t)(((sc + 2 * ng + 15) & m16) - (sc & m16));
            if constexpr (CK) {
              dst = ck_smem<CK>(W, dst, kARow, 4);
              if (csz > kARowCodes || ssz > kARow - kARowCodes) ck_record(5, csz << 16 | ssz);
            }
            bulk_g2s(dst, reinterpret_cast<const void *>(c & m16), csz, full);
            bulk_g2s(dst + kARowCodes, reinterpret_cast<const void *>(sc & m16),
                     ssz, full);
          }
        }
        if (lane == 0) ck_trace<CK>(trace, 0, t, ws, 2);
        ws = we;
        ++u;
        if (++s == P.code_stages) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    if (lane == 0) ck_trace<CK>(trace, 0, 0xFFFF, 0, 3);
    // no copy may still be landing in shared memory when the CTA exits
    // (after a time-out some fills are never consumed)
    if (lane == 0) {
      for (int j = u > P.code_stages ? u - P.code_stages : 0; j < u; ++j)
        mbar_wait(B0 + kBarCodeFull + 8 * (j % P.code_stages),
                  (uint32_t)(j / P.code_stages) & 1u);
    }
  } else if (warp == kWarpX) {
    // ---- x producer: the 128 k x n_pad tile of each iteration ---------------
    // (two copies of 64 k x n_pad rows, 128-byte rows with the 128-byte
    // swizzle: the K-major layout the MMA reads)
    if (lane == 0) {
      int s = 0, u = 0;
      uint32_t ph = 0;  // (u / x_stages) & 1, kept without a division
      bool ok = true;
      const uint32_t half = (uint32_t)n_pad * 128u;
      for (int t = cid; ok && t < P.tiles; t += nclusters) {
        for (int it = it0; it < it1; ++it) {
          if (u >= P.x_stages &&
              !mbar_wait(B0 + kBarXEmpty + 8 * s, ph ^ 1u, abort_addr, lim)) {
            if constexpr (CK) ck_record(22, (uint64_t)u);
            ok = false;
            break;
          }
          const uint32_t full = B0 + kBarXFull + 8 * s;
          const uint32_t dst = x_ring + (uint32_t)s * P.x_stage_bytes;
          const int k0 = (it < P.kblocks ? it : it % P.kblocks) * kKB;
          ck_trace<CK>(trace, 1, t, it, 1);
          mbar_arrive_expect_tx(full, 2u * half);
          for (int h = 0; h < 2; ++h) {
            uint32_t d = dst + (uint32_t)h * half;
            if constexpr (CK) {
              d = ck_smem<CK>(W, d, half, 6);
              if ((d & 1023u) != 0u) ck_record(7, d);
            }
            tma_load_2d(d, &tmap_x, k0 + 64 * h, 0, full);
          }
          ++u;
          if (++s == P.x_stages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      for (int j = u > P.x_stages ? u - P.x_stages : 0; j < u; ++j)
        mbar_wait(B0 + kBarXFull + 8 * (j % P.x_stages),
                  (uint32_t)(j / P.x_stages) & 1u);
    }
  } else if (warp == kWarpMma) {
    // ---- MMA issuer ---------------------------------------------------------
    // The whole warp follows the stages; lane 0 issues. The issuer touches
    // no shared memory while stages flow: the first shared-memory access
    // after a run of tcgen05.mma stalls until those MMAs complete, so the
    // waits on the input barriers belong to the waiter warp, which hands
    // each stage over through a named-barrier reduction (its vote says
    // whether the inputs arrived or a wait gave up).
    const uint32_t idesc = idesc_bf16_f32(kTileM, n_pad);
    const uint32_t xhalf = (uint32_t)n_pad * 128u;  // k 64..127 of the tile
    int xs = 0, ux = 0, as = 0, ua = 0;
    int ca = 0;  // accumulator commits
    bool ok = true;
    int i = 0;
    for (int t = cid; ok && t < P.tiles; t += nclusters, ++i) {
      const int buf = i & 1;
      const uint32_t d = tmem + (uint32_t)buf * kAccCols;
      for (int it = it0; it < it1; ++it) {
        ok = bar_red_and(kBarIdStage, 64, true);
        if (!ok) break;
        if (lane == 0) {
          tc_fence_after_sync();
          ck_trace<CK>(trace, 2, t, it, 1);
          const uint32_t xb = x_ring + (uint32_t)xs * P.x_stage_bytes;
          const uint32_t a = tmem + kAStage0 + (uint32_t)as * kAStageCols;
          if constexpr (CK) {
            if ((d & 0xFFFFu) + (uint32_t)n_pad > 2 * kAccCols || (d >> 16) != 0u)
              ck_record(8, d);
            if ((a & 0xFFFFu) + 128u > kTmemCols || (a >> 16) != 0u) ck_record(9, a);
            ck_smem<CK>(W, xb, P.x_stage_bytes, 10);
          }
#pragma unroll
          for (int k16 = 0; k16 < 8; ++k16) {
            const uint64_t bd = smem_desc_kmajor_sw128(
                xb + (uint32_t)(k16 >> 2) * xhalf + 32u * (uint32_t)(k16 & 3));
            mma_bf16_ts(d, a + 8u * (uint32_t)k16, bd, idesc,
                        (it > it0 || k16 > 0) ? 1u : 0u);
            if (!grid)
              mma_bf16_ts(d, a + 64u + 8u * (uint32_t)k16, bd, idesc, 1u);
          }
          mma_commit(B0 + kBarXEmpty + 8 * xs);
          mma_commit(B0 + kBarAEmpty + 8 * as);
        }
        __syncwarp();
        ++ux;
        xs = xs + 1 == P.x_stages ? 0 : xs + 1;
        ++ua;
        as = as + 1 == kAStages ? 0 : as + 1;
      }
      if (!ok) break;
      if (lane == 0) {
        ck_trace<CK>(trace, 2, t, 0, 2);
        mma_commit(B0 + kBarAccFull + 8 * buf);
        ck_trace<CK>(trace, 2, t, 0, 3);
      }
      __syncwarp();
      ++ca;
    }
    // The arrives of tcgen05.commit land asynchronously, when the MMAs
    // finish: before the CTA may leave (and its shared memory go to the
    // next CTA), every arrive this thread caused must have landed. The
    // drain commit covers every issued MMA; the last commit to each x and
    // A stage is then observed on its own barrier (those barriers complete
    // only through these commits). Bounded waits, also after a time-out.
    if (lane == 0) {
      mma_commit(B0 + kBarDrain);
      mbar_wait(B0 + kBarDrain, 0u);
      for (int j = ux > P.x_stages ? ux - P.x_stages : 0; j < ux; ++j)
        mbar_wait(B0 + kBarXEmpty + 8 * (j % P.x_stages),
                  (uint32_t)(j / P.x_stages) & 1u);
      for (int j = ua > kAStages ? ua - kAStages : 0; j < ua; ++j)
        mbar_wait(B0 + kBarAEmpty + 8 * (j % kAStages),
                  (uint32_t)(j / kAStages) & 1u);
      for (int j = ca > 2 ? ca - 2 : 0; j < ca; ++j)
        mbar_wait(B0 + kBarAccFull + 8 * (j & 1), (uint32_t)(j >> 1) & 1u);
    }
    __syncwarp();
  } else if (warp == kWarpWait) {
    // ---- waiter: the MMA issuer's input barriers ----------------------------
    // Per stage: the accumulator buffer is free (first stage of a tile, from
    // the third tile on), the x stage and the A stage are full; then one
    // named-barrier reduction with the issuer carries the verdict. Both
    // sides stop at the first failed stage, so they take the same number of
    // reductions.
    int xs = 0, ux = 0, as = 0, ua = 0;
    uint32_t xph = 0, aph = 0;  // phases of the x and A rings
    bool ok = true;
    int i = 0;
    for (int t = cid; ok && t < P.tiles; t += nclusters, ++i) {
      const int buf = i & 1;
      bool acc_ok = true;
      if (i >= 2)
        acc_ok = mbar_wait(B0 + kBarAccEmpty + 8 * buf,
                           (uint32_t)((i >> 1) + 1) & 1u, abort_addr, lim);
      if constexpr (CK) if (!acc_ok && lane == 0) ck_record(23, (uint64_t)i);
      for (int it = it0; it < it1; ++it) {
        bool got = acc_ok &&
                   mbar_wait(B0 + kBarXFull + 8 * xs, xph, abort_addr, lim) &&
                   mbar_wait(B0 + kBarAFull + 8 * as, aph, abort_addr, lim);
        got = __all_sync(0xFFFFFFFFu, got);
        if constexpr (CK) if (!got && lane == 0) ck_record(24, (uint64_t)ux << 32 | (uint32_t)ua);
        ok = bar_red_and(kBarIdStage, 64, got);
        if (!ok) break;
        ++ux;
        if (++xs == P.x_stages) {
          xs = 0;
          xph ^= 1u;
        }
        ++ua;
        if (++as == kAStages) {
          as = 0;
          aph ^= 1u;
        }
      }
    }
  } else if (warp < kWarpDec) {
    // ---- epilogue -----------------------------------------------------------
    const int q = warp & 3;  // tensor-memory lane quarter
    const int r = 32 * q + lane;
    bool dead = false;
    int i = 0;
    for (int t = cid; t < P.tiles; t += nclusters, ++i) {
      const int64_t row0 = (int64_t)t * kTileM;
      const int buf = i & 1;
      uint32_t v[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) v[c] = 0x7FC00000u;  // NaN unless read
      if (!dead) {
        const bool got = mbar_wait(B0 + kBarAccFull + 8 * buf,
                                   (uint32_t)(i >> 1) & 1u, abort_addr, lim);
        if constexpr (CK) if (!got) ck_record(25, (uint64_t)i);
        dead = !__all_sync(0xFFFFFFFFu, got);
        if (!dead) {
          tc_fence_after_sync();
          if (lane == 0) ck_trace<CK>(trace, 3 + (q == 0 ? 0 : 1) * 0, t, 0, 1 + 16 * q);
          const uint32_t ta =
              tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)buf * kAccCols;
          if constexpr (CK) ck_tmem<CK>(ta, (uint32_t)n_pad, (uint32_t)(32 * q), 11);
          __syncwarp();  // converged for the warp-wide loads
          tmem_ld16(ta, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
          if (n_pad > 16)
            tmem_ld16(ta + 16, *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
          if (n_pad > 32)
            tmem_ld16(ta + 32, *reinterpret_cast<uint32_t(*)[16]>(&v[32]));
          if (n_pad > 48)
            tmem_ld16(ta + 48, *reinterpret_cast<uint32_t(*)[16]>(&v[48]));
          tmem_ld_wait();
          if (lane == 0) ck_trace<CK>(trace, 4, t, 0, 2 + 16 * q);
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(B0 + kBarAccEmpty + 8 * buf);
        }
      }
      if (ks == 1) {
        // the whole K: this thread's row goes straight to y (NaN after a
        // time-out)
        const int64_t row = row0 + r;
        if (row < N) {
          float scale = 1.0f;
          if constexpr (FMT == TQ_FMT_B) {
            if (w.scales != nullptr)
              scale = __half2float(__ushort_as_half(w.scales[row / w.rps]));
          }
#pragma unroll
          for (int b = 0; b < 64; ++b)
            if (b < nb) {
              if constexpr (CK) {
                if (b >= batch) {
                  ck_record(12, (uint64_t)row);
                  continue;
                }
              }
              y[(int64_t)b * ldy + row] = scale * (unit * __uint_as_float(v[b]));
            }
        }
      } else {
        // a K slice: the partial tile goes to this CTA's shared buffer
        // (batch column c at part[c * 128 ..]: a warp's stores and the
        // owners' reads are 32 consecutive words, conflict-free), and the
        // cluster adds the ks partials through distributed shared memory,
        // each CTA the rows it owns, in rank order (deterministic). Per
        // tile, each CTA arrives once on every CTA's "part full" barrier
        // (its partial is written) and once on every CTA's "part free"
        // barrier (it has read the partials), so a buffer is overwritten
        // only after every peer has read it. A CTA whose epilogue stopped
        // (time-out) arrives no more: its peers' next wait times out, and
        // the rows of the tiles still open are NaN.
        const int et = (int)threadIdx.x - 32 * kWarpEpi;  // 0..127
        if (i >= 1 && !dead) {
          const bool got = mbar_wait_cluster(B0 + kBarPartFree,
                                             (uint32_t)(i - 1) & 1u,
                                             abort_addr, lim);
          if constexpr (CK) if (!got) ck_record(26, (uint64_t)i);
          dead = !got;
        }
        if constexpr (CK) ck_smem<CK>(W, P.red + delta, (uint32_t)(kTileM * n_pad * 4), 14);
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c < n_pad)
            part[c * kTileM + r] = dead ? __int_as_float(0x7FC00000)
                                        : __uint_as_float(v[c]);
        asm volatile("fence.acq_rel.cluster;" ::: "memory");
        dead = !bar_red_and(kBarIdEpi, 128, !dead);
        if (!dead && et == 0)
          for (int p = 0; p < ks; ++p)
            mbar_arrive_cluster(B0 + kBarPartFull, (uint32_t)p);
        bool full = false;
        if (!dead) {
          full = mbar_wait_cluster(B0 + kBarPartFull, (uint32_t)i & 1u,
                                   abort_addr, lim);
          if constexpr (CK) if (!full) ck_record(27, (uint64_t)i);
        }
        // this CTA's rows: 16-byte vectors (4 rows of one batch column) from
        // every CTA's partial tile, two vectors per thread in flight
        namespace cg = cooperative_groups;
        cg::cluster_group cluster = cg::this_cluster();
        const int own4 = (r_hi - r_lo) / 4;
        const int units = own4 * nb;
        for (int u0 = et; u0 < units; u0 += 256) {
          float4 acc[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float qn = __int_as_float(0x7FC00000);
            acc[h] = make_float4(qn, qn, qn, qn);
          }
          if (full) {
#pragma unroll
            for (int h = 0; h < 2; ++h) acc[h] = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int p = 0; p < ks; ++p) {
              const float *pp = cluster.map_shared_rank(part, p);
              float4 v4[2];
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int u = u0 + 128 * h;
                const int uu = u < units ? u : u0;
                const int g = uu % own4, b = uu / own4;
                v4[h] = *reinterpret_cast<const float4 *>(
                    pp + b * kTileM + r_lo + 4 * g);
              }
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                acc[h].x += v4[h].x;
                acc[h].y += v4[h].y;
                acc[h].z += v4[h].z;
                acc[h].w += v4[h].w;
              }
            }
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int u = u0 + 128 * h;
            if (u >= units) continue;
            const int g = u % own4, b = u / own4;
            const float sv[4] = {acc[h].x, acc[h].y, acc[h].z, acc[h].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int64_t row = row0 + r_lo + 4 * g + e;
              if (row < N) {
                float scale = 1.0f;
                if constexpr (FMT == TQ_FMT_B) {
                  if (w.scales != nullptr)
                    scale =
                        __half2float(__ushort_as_half(w.scales[row / w.rps]));
                }
                y[(int64_t)b * ldy + row] = scale * (unit * sv[e]);
              }
            }
          }
        }
        dead = !bar_red_and(kBarIdEpi, 128, full);
        if (!dead && et == 0)
          for (int p = 0; p < ks; ++p)
            mbar_arrive_cluster(B0 + kBarPartFree, (uint32_t)p);
      }
    }
  } else if (warp < kWarpDec + kDecWarps) {
    // ---- decoders -----------------------------------------------------------
    // One copy of the loop per decode variant, chosen once after the set-up:
    // while stages flow, only the running variant's code is fetched (the
    // variants together overflow the instruction cache).
    auto decoders = [&](auto dec_tag) {
      constexpr int DEC = decltype(dec_tag)::value;
      constexpr bool kB7 = DEC == kDecB7Grid || DEC == kDecB7Pair;
      constexpr bool kGrid =
          DEC == kDecGrid || DEC == kDecIdent || DEC == kDecB7Grid;
      const int q = warp & 3;
      const int kp = (warp - kWarpDec) >> 2;  // which 64-k half of the block
      const int r = 32 * q + lane;
      const uint32_t lane_tab =
          tab | (uint32_t)lane << (FMT == TQ_FMT_B ? 2 : 3);
      const uint32_t t_hi =
          tmem + ((uint32_t)(32 * q) << 16) + kAStage0 + 32u * (uint32_t)kp;
      const bool skip_first = P.skip_first_arrive != 0;
      int cs = 0, uc = 0, as = 0, ua = 0;
      uint32_t cph = 0, aph = 0;  // phases of the code and A rings
      bool ok = true;
      // this warp's compact book (adaptive alphabet)
      const uint32_t ctab = tab + (uint32_t)(warp - kWarpDec) * 1024u;
      for (int t = cid; ok && t < P.tiles; t += nclusters) {
        const int64_t row = (int64_t)t * kTileM + r;
        const bool row_ok = row < N;
        if constexpr (DEC == kDecAdaptive) {
          // rows t * 128 + 32 q .. + 31 share one book (lut_rows % 32 == 0);
          // a warp wholly past N reads book 0 (its weights are masked)
          const int64_t r0w = (int64_t)t * kTileM + 32 * q;
          const float *bl = w.lut + ((r0w < N ? r0w : 0) / w.lut_rows) * 256;
          __syncwarp();  // this warp's lookups of the previous tile are done
          for (int e = lane; e < 256; e += 32) {
            const float v = __ldg(bl + e);
            const uint32_t h = bf16_bits_rn(v);
            const uint32_t l = bf16_bits_rn(v - __uint_as_float(h << 16));
            asm volatile("st.shared.u32 [%0], %1;" ::"r"(ctab + 4u * (uint32_t)e),
                         "r"(h | l << 16)
                         : "memory");
          }
          __syncwarp();
        }
        for (int ws = it0; ws < it1;) {
          // Format B: one block per window (no division on the hot path)
          const int we =
              FMT == TQ_FMT_B ? ws + 1 : window_end(ws, it1, P.kblocks, kWin);
          ok = __all_sync(0xFFFFFFFFu, mbar_wait(B0 + kBarCodeFull + 8 * cs,
                                                 cph, abort_addr, lim));
          if constexpr (CK) if (!ok && lane == 0) ck_record(28, (uint64_t)uc);
          if (!ok) break;
          // this row's codes (crow) and scales (srow) in the stage; a row
          // written by a tensor copy is swizzled: logical byte o is at o ^ sw
          const bool swz = (FMT == TQ_FMT_B && !kB7) || P.a_map;
          const uint32_t sw = swz ? (uint32_t)(r & 7) << 4 : 0u;
          const uint32_t crow =
              code_stage(cs) +
              (uint32_t)r * (FMT == TQ_FMT_B ? (kB7 ? kB7Row : kBRow)
                             : swz           ? kARowCodes
                                             : kARow);
          const uint32_t srow = swz ? code_stage(cs) + kAMapScales +
                                          (uint32_t)r * kAMapSRow
                                    : crow + kARowCodes;
          // Format A: byte skews of the window's first group inside the code and
          // scale rows (the same for every row with tensor copies)
          uint32_t cskew = 0, sskew = 0;
          int64_t g0 = 0;
          if constexpr (FMT == TQ_FMT_A) {
            const int plane = ws / P.kblocks;
            g0 = 2 * (int64_t)(ws - plane * P.kblocks);
            if (swz) {
              cskew = (uint32_t)(13 * g0) & 15u;
              sskew = 2u * ((uint32_t)g0 & 7u);
            } else {
              const int64_t gi = (row_ok ? row : 0) * gpr + g0;
              cskew = (uint32_t)((reinterpret_cast<uintptr_t>(w.codes) +
                                  (uintptr_t)(plane * w.codes_plane_stride) +
                                  (uintptr_t)(gi * 13)) &
                                 15);
              sskew = (uint32_t)((reinterpret_cast<uintptr_t>(w.scales) +
                                  (uintptr_t)(2 * (plane * w.scales_plane_stride +
                                                   gi))) &
                                 15);
            }
          }
          for (int it = ws; it < we; ++it) {
            if (ua >= kAStages) {
              ok = __all_sync(0xFFFFFFFFu,
                              mbar_wait(B0 + kBarAEmpty + 8 * as, aph ^ 1u,
                                        abort_addr, lim));
              if constexpr (CK) if (!ok && lane == 0) ck_record(29, (uint64_t)ua);
              if (!ok) break;
            }
            tc_fence_after_sync();
            if (lane == 0 && q == 0 && kp == 0) ck_trace<CK>(trace, 5, t, it, 1);
            uint32_t hi[32], lo[32];
            uint32_t ta = t_hi + (uint32_t)as * kAStageCols;
            if constexpr (CK) ta = ck_tmem<CK>(ta, 96u, (uint32_t)(32 * q), 19);
            if constexpr (FMT == TQ_FMT_B && DEC == kDecIdent) {
              // table-free decode in 4 chunks of 16 codes, each stored to
              // tensor memory (8 columns) at once: a short loop body keeps
              // the decoder's hot code small. An invalid code poisons its
              // chunk (NaN operands), which poisons the row's sums; k past
              // K (in the last block) and rows past N get zero weights.
              const int64_t kv = K - ((int64_t)it * kKB + 64 * kp);
              const bool edge = __any_sync(0xFFFFFFFFu, kv < 64 || !row_ok);
#pragma unroll 1
              for (int j = 0; j < 4; ++j) {
                const uint32_t a =
                    crow + ((64u * (uint32_t)kp + 16u * (uint32_t)j) ^ sw);
                uint32_t h8[8];
                if (decode_b_arith16(lds128(ck_smem<CK>(W, a, 16u, 16)), h8) !=
                    0u) {
#pragma unroll
                  for (int m = 0; m < 8; ++m) h8[m] = 0x7FC07FC0u;
                }
                if (edge) {
#pragma unroll
                  for (int m = 0; m < 8; ++m) {
                    const uint32_t keep =
                        (row_ok && 2 * (8 * j + m) < kv) ? 0xFFFFFFFFu : 0u;
                    h8[m] &= keep;
                  }
                }
                __syncwarp();  // converged for the warp-wide store
                tmem_st8(ta + 8u * (uint32_t)j, h8);
              }
            } else if constexpr (FMT == TQ_FMT_B) {
              // this half's 64 codes: four 16-byte loads. 7-bit alphabet: 56
              // bytes, loaded from byte 0 (kp 0) or 48 (kp 1, the run starting
              // 8 bytes in); its row pitch, 112, puts a quarter warp's 8 rows
              // on 8 distinct 16-byte bank groups
              const uint32_t hoff = (kB7 ? 48u : 64u) * (uint32_t)kp;
              uint32_t cw[16];
  #pragma unroll
              for (int j = 0; j < 4; ++j) {
                const uint32_t a = crow + ((hoff + 16u * (uint32_t)j) ^ sw);
                const uint4 v4 = lds128(ck_smem<CK>(W, a, 16u, 16));
                cw[4 * j] = v4.x;
                cw[4 * j + 1] = v4.y;
                cw[4 * j + 2] = v4.z;
                cw[4 * j + 3] = v4.w;
              }
              if constexpr (kB7) {
                uint32_t d[14];
  #pragma unroll
                for (int i = 0; i < 14; ++i) d[i] = kp ? cw[i + 2] : cw[i];
                decode_b7<!kGrid>(d, lane_tab, hi, lo);
              } else if constexpr (DEC == kDecAdaptive) {
                decode_b_compact(cw, ctab, hi, lo);
              } else if constexpr (DEC == kDecGrid) {
                decode_b_hi(cw, lane_tab, hi);
              } else {
                decode_b(cw, lane_tab, hi, lo);
              }
              // k past K (in the last block) and rows past N: zero weights
              // (selects, no branch: the tcgen05.st below is warp-wide)
              const int64_t kv = K - ((int64_t)it * kKB + 64 * kp);
              if (__any_sync(0xFFFFFFFFu, kv < 64 || !row_ok)) {
  #pragma unroll
                for (int m = 0; m < 32; ++m) {
                  const uint32_t keep = (row_ok && 2 * m < kv) ? 0xFFFFFFFFu : 0u;
                  hi[m] &= keep;
                  if constexpr (!kGrid) lo[m] &= keep;
                }
              }
            } else {
              const int gi = 2 * (it - ws) + kp;  // group inside the window
              const bool valid = row_ok && g0 + gi < gpr;
              const uint32_t o = cskew + 13u * (uint32_t)gi;
              const uint32_t wl = o & ~3u;  // logical offsets wl .. wl + 15
              const uint32_t sh = 8u * (o & 3u);
              const uint32_t w0 = lds32(ck_smem<CK>(W, crow + (wl ^ sw), 4u, 17)),
                             w1 = lds32(ck_smem<CK>(W, crow + ((wl + 4) ^ sw), 4u, 17)),
                             w2 = lds32(ck_smem<CK>(W, crow + ((wl + 8) ^ sw), 4u, 17)),
                             w3 = lds32(ck_smem<CK>(W, crow + ((wl + 12) ^ sw), 4u, 17));
              const uint32_t b[4] = {__funnelshift_r(w0, w1, sh),
                                     __funnelshift_r(w1, w2, sh),
                                     __funnelshift_r(w2, w3, sh), w3 >> sh};
              const uint32_t sa = srow + sskew + 2u * (uint32_t)gi;
              const uint32_t sbits =
                  (lds32(ck_smem<CK>(W, sa & ~3u, 4u, 18)) >> (8u * (sa & 2u))) & 0xFFFFu;
              const float sf = __half2float(__ushort_as_half((unsigned short)sbits));
              const uint32_t h = bf16_bits_rn(sf);
              const uint32_t l = bf16_bits_rn(sf - __uint_as_float(h << 16));
              decode_a(b, lane_tab, h ^ 0x8000u, h, l ^ 0x8000u, l, hi, lo);
              if (__any_sync(0xFFFFFFFFu, !valid)) {
                const uint32_t keep = valid ? 0xFFFFFFFFu : 0u;
  #pragma unroll
                for (int m = 0; m < 32; ++m) {
                  hi[m] &= keep;
                  lo[m] &= keep;
                }
              }
            }
            if constexpr (!(FMT == TQ_FMT_B && DEC == kDecIdent)) {
              __syncwarp();  // converged for the warp-wide stores
              tmem_st32(ta, hi);
              if constexpr (!kGrid) tmem_st32(ta + 64u, lo);
            }
            tmem_st_wait();
            if (lane == 0 && q == 0 && kp == 0) ck_trace<CK>(trace, 5, t, it, 2);
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0 && !(skip_first && ua == 0))
              mbar_arrive(B0 + kBarAFull + 8 * as);
            ++ua;
            if (++as == kAStages) {
              as = 0;
              aph ^= 1u;
            }
          }
          if (!ok) break;
          // this warp is done reading the window
          __syncwarp();
          if (lane == 0) mbar_arrive(B0 + kBarCodeEmpty + 8 * cs);
          ws = we;
          ++uc;
          if (++cs == P.code_stages) {
            cs = 0;
            cph ^= 1u;
          }
        }
      }
    };
    if constexpr (FMT == TQ_FMT_B) {
      if (b7) {
        if (grid)
          decoders(std::integral_constant<int, kDecB7Grid>{});
        else
          decoders(std::integral_constant<int, kDecB7Pair>{});
      } else if (adaptive) {
        decoders(std::integral_constant<int, kDecAdaptive>{});
      } else if (ident) {
        decoders(std::integral_constant<int, kDecIdent>{});
      } else if (grid) {
        decoders(std::integral_constant<int, kDecGrid>{});
      } else {
        decoders(std::integral_constant<int, kDecPair>{});
      }
    } else {
      decoders(std::integral_constant<int, kDecPair>{});
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (threadIdx.x == 0) ck_trace<CK>(trace, 6, 0xFFFF, 0, 1);
  // every CTA of a cluster stays until its peers have read its partials and
  // arrived on its barriers
  if (ks > 1) {
    __syncwarp();
    cooperative_groups::this_cluster().sync();
  }
  if (warp == kWarpMma) {
    __syncwarp();  // converged for the warp-wide free
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
    if (lane == 0) ck_trace<CK>(trace, 7, 0xFFFF, 0, 1);
  }
}

// ---- host side ---------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault,
                                &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Shared-memory plan for clusters of `ks`; false if it does not fit. The
// dynamic window starts at `base` (the per-CTA reserved shared memory).
bool plan_smem(int fmt, int n_pad, int ks, uint32_t base, TcPlan *P) {
  P->n_pad = n_pad;
  P->ks = ks;
  P->base = base;
  const uint32_t end = base + (uint32_t)kSmemMax;
  const uint32_t tab = (base + 0xFFFFu) & ~0xFFFFu;
  if (tab + 0x10000u > end) return false;
  P->tab = tab;
  P->code_stage_bytes = kTileM * (fmt == TQ_FMT_B ? kBRow : kARow);
  P->x_stage_bytes = (uint32_t)n_pad * kKB * 2u;
  P->x_stages = n_pad <= 32 ? kMaxXStages : 3;
  // with a split of K, every CTA keeps its partial tile [n_pad][128] fp32
  const uint32_t red_bytes = ks > 1 ? (uint32_t)(kTileM * n_pad * 4) : 0u;
  // below the table: code stages (1024-byte aligned: the 128-byte swizzle
  // of tensor copies repeats every 8 rows of 128 bytes)
  const uint32_t lo0 = (base + 1023u) & ~1023u;
  P->code_lo = lo0;
  P->code_lo_n = (int)((tab - lo0) / P->code_stage_bytes);
  // above it: barriers, x ring, reduction buffer, further code stages
  uint32_t a = tab + 0x10000u;
  P->bars = a;
  a += kBarBytes;
  a = (a + 1023u) & ~1023u;  // 128-byte swizzle atoms
  P->x_ring = a;
  a += (uint32_t)P->x_stages * P->x_stage_bytes;
  P->red = a;
  a += red_bytes;
  a = (a + 1023u) & ~1023u;
  P->code_hi = a;
  if (a > end) return false;
  int hi_n = (int)((end - a) / P->code_stage_bytes);
  if (P->code_lo_n > kMaxCodeStages) P->code_lo_n = kMaxCodeStages;
  if (P->code_lo_n + hi_n > kMaxCodeStages) hi_n = kMaxCodeStages - P->code_lo_n;
  P->code_stages = P->code_lo_n + hi_n;
  if (P->code_stages < 2) return false;
  const uint32_t top = hi_n > 0
                           ? P->code_hi + (uint32_t)hi_n * P->code_stage_bytes
                           : P->red + red_bytes;
  P->smem = (size_t)(top - base);
  return P->smem <= (size_t)kSmemMax;
}

// Clusters of `ks` CTAs (one per SM) that can be resident together.
int resident_clusters(const void *kern, int ks, size_t smem) {
  // An error already pending belongs to the caller: leave it and skip.
  if (cudaPeekAtLastError() != cudaSuccess) return 0;
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
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();  // the query's own error
    return 0;
  }
  return n;
}

template <int FMT, bool CK>
cudaError_t launch_tc_as(const WeightsView &w, const __nv_bfloat16 *x,
                      int64_t batch, int64_t ldx, float *y, int64_t ldy,
                      cudaStream_t stream) {
  auto kern = gemm_tc_kernel<FMT, CK>;
  cudaError_t e = ensure_smem_limit<gemm_tc_kernel<FMT, CK>>(kSmemMax);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148, reserved = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock,
                             dev);
  if (e != cudaSuccess) return e;
  const int n_pad = (int)((batch + 15) / 16 * 16);
  const int kblocks = (int)((w.k + kKB - 1) / kKB);
  const int iters = (FMT == TQ_FMT_A ? w.planes : 1) * kblocks;
  const int64_t tiles = (w.n + kTileM - 1) / kTileM;
  if (tiles > (1 << 30) || iters < 1) return cudaErrorInvalidValue;

  // Cluster size: the K split whose resident clusters finish the tiles with
  // the fewest iterations per CTA (ceil(tiles / resident clusters) tiles of
  // ceil(iters / ks) blocks, plus a set-up allowance), preferring no split.
  static std::atomic<int> occ_cache[16][2][4][9];  // per instantiation
  TcPlan best{};
  int best_clusters = 0;
  int64_t best_cost = -1;
  const int force_ks = g_test_tc_ks.load(), max_clusters = g_test_tc_clusters.load();
  for (int ks = 1; ks <= 8 && ks <= iters; ++ks) {
    if (force_ks > 0 && ks != force_ks) continue;
    TcPlan P{};
    if (!plan_smem(FMT, n_pad, ks, (uint32_t)reserved, &P)) continue;
    std::atomic<int> *slot =
        dev < 16 ? &occ_cache[dev][FMT - 1][n_pad / 16 - 1][ks] : nullptr;
    int c = slot ? slot->load() : 0;
    if (c <= 0) {
      c = resident_clusters(reinterpret_cast<const void *>(kern), ks, P.smem);
      if (c <= 0 && ks == 1) c = sms;
      if (slot && c > 0) slot->store(c);
    }
    if (c <= 0) continue;
    // persistent clusters walk the tiles (with a split, each tile's partials
    // are added while the next tile runs); the set-up and the last tile's
    // epilogue are paid once. Measured on B200: when clusters of 3, 5, 6 or
    // 7 CTAs walk several tiles, every further tile costs about 4 blocks
    // more (the per-tile hand-over between the CTAs is exposed; clusters of
    // 2, 4 and 8 hide it)
    int64_t clusters = c < tiles ? c : tiles;
    if (max_clusters > 0 && clusters > max_clusters) clusters = max_clusters;
    const int64_t waves = (tiles + clusters - 1) / clusters;
    const bool pow2 = (ks & (ks - 1)) == 0;
    const int64_t cost = waves * (((int64_t)iters + ks - 1) / ks) +
                         (ks == 1 ? 2 : 4) + (pow2 ? 0 : 4 * (waves - 1));
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = P;
      best_clusters = (int)clusters;
    }
  }
  if (best_cost < 0) return cudaErrorInvalidConfiguration;
  best.tiles = (int)tiles;
  best.kblocks = kblocks;
  best.iters = iters;
  const uint64_t tw = g_test_wait_ns.load();
  best.wait_ns = tw ? tw : kWaitLimitNs;
  best.skip_first_arrive = g_test_skip_first_arrive.load();
  best.grid_ok = g_test_force_path.load() == 3 ? 0 : 1;

  auto encode = encode_fn();
  if (encode == nullptr) return cudaErrorNotSupported;
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  // x: K bf16 per row, `batch` rows ldx apart; boxes of 64 k x n_pad rows
  // (128-byte rows, 128-byte swizzle). Rows past the batch and k past K
  // read as zero.
  CUtensorMap tmap_x;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)w.k, (cuuint64_t)batch};
    const cuuint64_t strides[1] = {(cuuint64_t)ldx * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)n_pad};
    if (encode(&tmap_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
               const_cast<__nv_bfloat16 *>(x), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  // codes (and Format A scales)
  CUtensorMap tmap_c, tmap_s;
  memset(&tmap_c, 0, sizeof(tmap_c));
  memset(&tmap_s, 0, sizeof(tmap_s));
  best.a_map = 0;
  if (FMT == TQ_FMT_B && w.format == TQ_FMT_B7) {
    // [N][7 K / 8] bytes (K a multiple of 128, so every row starts on a
    // 16-byte boundary); boxes of 128 rows x 112 bytes, not swizzled
    const cuuint64_t pitch = (cuuint64_t)(w.k / 128) * kB7Row;
    const cuuint64_t dims[2] = {pitch, (cuuint64_t)w.n};
    const cuuint64_t strides[1] = {pitch};
    const cuuint32_t box[2] = {kB7Row, (cuuint32_t)kTileM};
    if (encode(&tmap_c, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
               const_cast<uint8_t *>(w.codes), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else if (FMT == TQ_FMT_B) {
    // [N][K] bytes; boxes of 128 rows x 128 codes, 128-byte swizzle
    const cuuint64_t dims[2] = {(cuuint64_t)w.k, (cuuint64_t)w.n};
    const cuuint64_t strides[1] = {(cuuint64_t)w.k};
    const cuuint32_t box[2] = {kBRow, (cuuint32_t)kTileM};
    if (encode(&tmap_c, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
               const_cast<uint8_t *>(w.codes), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    // [plane][N][13 K/64] bytes and [plane][N][K/64] fp16 as 3-D tensors,
    // when every row and plane starts on a 16-byte boundary (K a multiple
    // of 1024); otherwise the producer copies each row's run by itself
    const int64_t gpr = w.k / 64;
    const int64_t cpitch = 13 * gpr, spitch = 2 * gpr;
    const int64_t cps = w.codes_plane_stride, sps = 2 * w.scales_plane_stride;
    if (cpitch % 16 == 0 && spitch % 16 == 0 &&
        (w.planes == 1 || (cps % 16 == 0 && sps % 16 == 0))) {
      const cuuint64_t cd[3] = {(cuuint64_t)cpitch, (cuuint64_t)w.n,
                                (cuuint64_t)w.planes};
      const cuuint64_t cs[2] = {(cuuint64_t)cpitch,
                                (cuuint64_t)(w.planes > 1 ? cps : cpitch * w.n)};
      const cuuint32_t cb[3] = {kARowCodes, (cuuint32_t)kTileM, 1u};
      const cuuint64_t sd[3] = {(cuuint64_t)gpr, (cuuint64_t)w.n,
                                (cuuint64_t)w.planes};
      const cuuint64_t ss[2] = {(cuuint64_t)spitch,
                                (cuuint64_t)(w.planes > 1 ? sps : spitch * w.n)};
      const cuuint32_t sb[3] = {kAMapSRow / 2, (cuuint32_t)kTileM, 1u};
      if (encode(&tmap_c, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
                 const_cast<uint8_t *>(w.codes), cd, cs, cb, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS &&
          encode(&tmap_s, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3,
                 const_cast<uint16_t *>(w.scales), sd, ss, sb, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
        best.a_map = 1;
    }
  }

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(best_clusters * best.ks), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = best.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)best.ks;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // programmatic dependent launch: the set-up and the first L2 prefetches
  // overlap the end of the kernel before (the kernel waits for it before
  // reading user memory)
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  unsigned long long *trace =
      CK ? reinterpret_cast<unsigned long long *>(g_test_trace.load()) : nullptr;
  return cudaLaunchKernelEx(&cfg, kern, w, batch, y, ldy, best, tmap_x, tmap_c,
                            tmap_s, trace);
}

template <int FMT>
cudaError_t launch_tc(const WeightsView &w, const __nv_bfloat16 *x,
                      int64_t batch, int64_t ldx, float *y, int64_t ldy,
                      cudaStream_t stream) {
  if (g_test_self_check.load() != 0)
    return launch_tc_as<FMT, true>(w, x, batch, ldx, y, ldy, stream);
  return launch_tc_as<FMT, false>(w, x, batch, ldx, y, ldy, stream);
}

}  // namespace

cudaError_t tc_check_record(uint64_t out[4], bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(out, g_tc_check, sizeof(g_tc_check));
  if (e != cudaSuccess || !reset) return e;
  const unsigned long long zero[4] = {0, 0, 0, 0};
  return cudaMemcpyToSymbol(g_tc_check, zero, sizeof(zero));
}

bool gemm_tc_supported(const WeightsView &w, int64_t batch) {
  // tensor-copy coordinates are 32-bit
  if (batch < 1 || w.k < 1 || w.n >= (1ll << 31) || w.k >= (1ll << 31))
    return false;
  // adaptive alphabet: a decoder warp's 32 rows must share a code book
  if (w.format == TQ_FMT_B) return w.lut_rows % 32 == 0;
  // 7-bit alphabet: tensor copies of whole 112-byte runs (128 indices) need
  // K a multiple of 128 and the codes on a 16-byte boundary
  if (w.format == TQ_FMT_B7)
    return w.k % 128 == 0 &&
           (reinterpret_cast<uintptr_t>(w.codes) & 15u) == 0;
  return w.format == TQ_FMT_A && w.group == 64;
}

cudaError_t gemm_tc(const WeightsView &w, const __nv_bfloat16 *x,
                    int64_t batch, int64_t ldx, float *y, int64_t ldy,
                    cudaStream_t stream) {
  for (int64_t b0 = 0; b0 < batch; b0 += kMaxN) {
    const int64_t nb = batch - b0 < kMaxN ? batch - b0 : kMaxN;
    const cudaError_t e =
        w.format == TQ_FMT_B || w.format == TQ_FMT_B7
            ? launch_tc<TQ_FMT_B>(w, x + b0 * ldx, nb, ldx, y + b0 * ldy, ldy,
                                  stream)
            : launch_tc<TQ_FMT_A>(w, x + b0 * ldx, nb, ldx, y + b0 * ldy, ldy,
                                  stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace tq
