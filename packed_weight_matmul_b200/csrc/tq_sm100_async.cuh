// sm_100 asynchronous-copy and synchronisation primitives used by the fused
// GEMM: shared-memory mbarriers, 1-D bulk copies and 2-D tensor copies (the
// TMA engine) global -> shared. Written from the PTX ISA descriptions of
// mbarrier, cp.async.bulk and cp.async.bulk.tensor.
//
// Every wait is bounded: it polls with try_wait until the barrier phase
// completes, a shared abort word becomes non-zero, or a time limit
// (%globaltimer, nanoseconds) passes, and reports which happened, so a kernel
// can never spin forever.
#pragma once

#include <stdint.h>

namespace tq {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count)
               : "memory");
}

// Make barrier initialisation visible to the async proxy and to the cluster.
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar)
               : "memory");
}

// Arrive and add `bytes` to the transaction count of the current phase.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar,
                                                      uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
                   bar),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with acquire at cluster scope: the writes that other CTAs of the
// cluster released with their arrivals are visible afterwards.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar,
                                                      uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Arrive, with release at cluster scope, on the barrier at this CTA's shared
// address `bar` in the cluster's CTA `rank` (the same offset in its window).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar,
                                                    uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
               : "=r"(remote)
               : "r"(bar), "r"(rank));
  asm volatile(
      "mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(
          remote)
      : "memory");
}

__device__ __forceinline__ int ld_volatile_s32(uint32_t addr) {
  int v;
  asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ void st_volatile_s32(uint32_t addr, int v) {
  asm volatile("st.volatile.shared.u32 [%0], %1;" ::"r"(addr), "r"(v)
               : "memory");
}

__device__ __forceinline__ void atom_min_shared_u32(uint32_t addr, uint32_t v) {
  asm volatile("atom.shared.min.u32 _, [%0], %1;" ::"r"(addr), "r"(v)
               : "memory");
}

// Wait for the phase with the given parity to complete. Returns false when
// the wait gave up: the word at `abort_addr` became non-zero, or `limit_ns`
// passed (then the abort word is set, so that the CTA's other roles stop).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          uint32_t abort_addr,
                                          uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (ld_volatile_s32(abort_addr) != 0) return false;
    if (global_ns() - t0 > limit_ns) {
      st_volatile_s32(abort_addr, 1);
      return false;
    }
  }
}

// As mbar_wait, with acquire at cluster scope (see mbar_try_wait_cluster).
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar,
                                                  uint32_t parity,
                                                  uint32_t abort_addr,
                                                  uint64_t limit_ns) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if (ld_volatile_s32(abort_addr) != 0) return false;
    if (global_ns() - t0 > limit_ns) {
      st_volatile_s32(abort_addr, 1);
      return false;
    }
  }
}

// Wait without an abort word (kernels with a single waiting role).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

// Bulk copy of `bytes` (multiple of 16; both addresses 16-byte aligned) from
// global to this CTA's shared memory, completing on `bar` as transaction
// bytes.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src,
                                         uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// 2-D tensor copy of one box (coordinates c0 innermost, c1) into this CTA's
// shared memory, completing on `bar`; out-of-range elements read as zero.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void *tmap,
                                            int32_t c0, int32_t c1,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::"
      "bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(tmap), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

// 3-D tensor copy of one box (coordinates c0 innermost, c1, c2) into this
// CTA's shared memory, completing on `bar`; out-of-range elements read as
// zero.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void *tmap,
                                            int32_t c0, int32_t c1, int32_t c2,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::"
      "bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

// ---- thread-block clusters -------------------------------------------------

// L2 prefetch of the box of a 2-D tensor map at (c0, c1) (no shared-memory
// destination, no barrier).
__device__ __forceinline__ void tma_prefetch_2d(const void *tmap, int c0,
                                                int c1) {
  asm volatile(
      "cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
          tmap),
      "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

}  // namespace tq
